// ep.cu -- expert parallelism: the experts are split over `world` ranks, and
// each rank's routed (token, expert) pairs travel to the rank that owns the
// expert and back.
//
// The GC-MoE abstract runs the MoE layer with its experts partitioned over
// GPUs, tokens dispatched to the GPU of their experts and the expert outputs
// combined back. Here each step is a kernel that writes straight into
// another rank's buffers through pointers the caller passes (buffers of the
// same GPU, or of a peer GPU with peer access enabled: the stores then cross
// NVLink). No step waits on another rank inside a kernel; the caller orders
// the phases (count -> dispatch -> local GEMMs -> combine -> finalize) with a
// barrier between ranks after count, dispatch and combine.
//
// Layout of rank d's receive buffer: rows grouped by d's local expert, and
// inside an expert by source rank, and inside a source by the source's
// permutation order (ascending pair id): the permuted-rows layout the grouped
// GEMMs take, with offsets from moe_ep_local_offsets. Every row keeps its
// origin (source rank, pair id), so combine puts its down output back at the
// source's pair id and the source's finalize runs with the identity
// permutation: the arithmetic of every pair is that of moe_forward on the
// source's own tokens.
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"

namespace moe {
namespace {

constexpr int kEpThreads = 256;
constexpr int kSrcShift = 24;               // recv_src entry: source rank << 24 | pair id

struct EpPtrs {
    int32_t *counts[MOE_EP_MAX_RANKS];
    uint16_t *recv_rows[MOE_EP_MAX_RANKS];
    int32_t *recv_src[MOE_EP_MAX_RANKS];
    uint16_t *y_ret[MOE_EP_MAX_RANKS];
    int pairs[MOE_EP_MAX_RANKS];
};

EpPtrs ptrs_of(const moe_ep_peers_t *p) {
    EpPtrs e;
    for (int r = 0; r < MOE_EP_MAX_RANKS; ++r) {
        e.counts[r] = p->counts[r];
        e.recv_rows[r] = p->recv_rows[r];
        e.recv_src[r] = p->recv_src[r];
        e.y_ret[r] = p->y_ret[r];
        e.pairs[r] = p->pairs[r];
    }
    return e;
}

// This rank's pairs per expert, into row `rank` of every owner's count matrix
// (zeros for a rank without tokens, whose offsets are never written).
__global__ void __launch_bounds__(kEpThreads) ep_count_kernel(const int32_t *__restrict__ offsets, int P, int E,
                                                             int E_loc, int rank, int world,
                                                             const __grid_constant__ EpPtrs p) {
    griddep_wait();
    for (int e = threadIdx.x; e < E; e += kEpThreads) {
        const int d = e / E_loc, el = e - d * E_loc;
        p.counts[d][rank * E_loc + el] = P > 0 ? offsets[e + 1] - offsets[e] : 0;
    }
}

// base[e] = start of this rank's rows of expert e in its owner's receive
// buffer: all rows of the owner's lower experts, then the lower ranks' rows
// of e. One exclusive scan over the E experts' totals over all ranks,
// restarted at each owner's first expert. Every thread of the CTA calls it;
// prefix is scratch of E ints.
__device__ void dest_bases(const EpPtrs &p, int E, int E_loc, int rank, int world, int *prefix, int *base) {
    __shared__ int chunk_sum[kEpThreads];
    const int per = (E + kEpThreads - 1) / kEpThreads;     // experts per thread, contiguous
    const int e0 = threadIdx.x * per;
    int run = 0;
    for (int i = 0; i < per && e0 + i < E; ++i) {
        const int e = e0 + i, d = e / E_loc, el = e - d * E_loc;
        int t = 0, below = 0;
        for (int s = 0; s < world; ++s) {
            const int c = p.counts[d][s * E_loc + el];
            t += c;
            if (s < rank) below += c;
        }
        prefix[e] = t;                                      // the total, for now
        base[e] = below;
        run += t;
    }
    chunk_sum[threadIdx.x] = run;
    __syncthreads();
    if (threadIdx.x == 0) {                                 // exclusive scan of the threads' sums
        int acc = 0;
        for (int i = 0; i < kEpThreads; ++i) {
            const int v = chunk_sum[i];
            chunk_sum[i] = acc;
            acc += v;
        }
    }
    __syncthreads();
    int excl = chunk_sum[threadIdx.x];
    for (int i = 0; i < per && e0 + i < E; ++i) {
        const int t = prefix[e0 + i];
        prefix[e0 + i] = excl;
        excl += t;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kEpThreads) base[e] += prefix[e] - prefix[(e / E_loc) * E_loc];
    __syncthreads();
}

// Row r of this rank's permutation (expert e, i-th of e's rows) -> row
// dest_base(e) + i of e's owner: the token's hidden row and its origin.
// One warp per row, 16-byte vectors.
__global__ void __launch_bounds__(kEpThreads) ep_dispatch_kernel(const uint4 *__restrict__ hidden,
                                                                const int32_t *__restrict__ perm,
                                                                const int32_t *__restrict__ offsets, int P, int K,
                                                                int vpr, int E, int E_loc, int rank, int world,
                                                                int capacity, const __grid_constant__ EpPtrs p, int *err) {
    extern __shared__ int ep_smem[];
    int *off_s = ep_smem;              // [E + 1]
    int *base_s = off_s + E + 1;       // [E]
    int *prefix_s = base_s + E;        // [E]
    griddep_wait();
    for (int e = threadIdx.x; e <= E; e += kEpThreads) off_s[e] = offsets[e];
    dest_bases(p, E, E_loc, rank, world, prefix_s, base_s);
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (kEpThreads / 32);
    for (int r = blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5); r < P; r += warps) {
        int lo = 0, hi = E - 1;                  // the expert whose segment holds row r
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off_s[mid] <= r) lo = mid; else hi = mid - 1;
        }
        const int e = lo, d = e / E_loc;
        const int dst = base_s[e] + (r - off_s[e]);
        const int pair = perm[r];
        if (dst < 0 || dst >= capacity || pair < 0 || pair >= P) {
            if (lane == 0) raise_error(err, kErrBounds);
            continue;
        }
        const uint4 *src = hidden + static_cast<size_t>(pair / K) * vpr;
        uint4 *out = reinterpret_cast<uint4 *>(p.recv_rows[d]) + static_cast<size_t>(dst) * vpr;
        for (int v = lane; v < vpr; v += 32) out[v] = __ldg(src + v);
        if (lane == 0) p.recv_src[d][dst] = (rank << kSrcShift) | pair;
    }
}

// Offsets of this rank's receive buffer over its local experts (one CTA).
__global__ void __launch_bounds__(kEpThreads) ep_offsets_kernel(const int32_t *__restrict__ counts, int E_loc,
                                                               int world, int32_t *__restrict__ offsets) {
    griddep_wait();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int el = 0; el < E_loc; ++el) {
            offsets[el] = run;
            for (int s = 0; s < world; ++s) run += counts[s * E_loc + el];
        }
        offsets[E_loc] = run;
    }
}

// Each received row's down output back to its source, at its pair id.
__global__ void __launch_bounds__(kEpThreads) ep_combine_kernel(const uint4 *__restrict__ y,
                                                               const int32_t *__restrict__ own_src,
                                                               const int32_t *__restrict__ offsets_local, int E_loc,
                                                               int vpr, int rank, int world,
                                                               const __grid_constant__ EpPtrs p, int *err) {
    griddep_wait();
    const int n = offsets_local[E_loc];
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (kEpThreads / 32);
    for (int i = blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5); i < n; i += warps) {
        const int code = own_src[i];
        const int s = code >> kSrcShift, pair = code & ((1 << kSrcShift) - 1);
        uint16_t *dst_rows = p.y_ret[0];
        int dst_pairs = p.pairs[0];
#pragma unroll
        for (int q = 1; q < MOE_EP_MAX_RANKS; ++q)
            if (q == s) {
                dst_rows = p.y_ret[q];
                dst_pairs = p.pairs[q];
            }
        if (s < 0 || s >= world || pair >= dst_pairs) {
            if (lane == 0) raise_error(err, kErrBounds);
            continue;
        }
        const uint4 *src = y + static_cast<size_t>(i) * vpr;
        uint4 *out = reinterpret_cast<uint4 *>(dst_rows) + static_cast<size_t>(pair) * vpr;
        for (int v = lane; v < vpr; v += 32) out[v] = src[v];
    }
}

int ep_grid(long long rows) {
    const long long per_cta = kEpThreads / 32;
    long long b = (rows + per_cta - 1) / per_cta;
    if (b > 148LL * 8) b = 148LL * 8;
    return b < 1 ? 1 : static_cast<int>(b);
}

// The checks every EP entry point makes; E_loc out.
moe_status_t check_ep(const moe_shape_t *s, const moe_ep_peers_t *p, int &E_loc) {
    moe_status_t st = validate_shape(s);
    if (st != MOE_OK) return st;
    if (!p || p->world < 1 || p->world > MOE_EP_MAX_RANKS || p->rank < 0 || p->rank >= p->world || p->capacity < 0)
        return MOE_ERR_INVALID_ARG;
    if (s->n_shared != 0 || s->E % p->world) return MOE_ERR_UNSUPPORTED;
    if (s->fmt != MOE_W_BF16 && s->fmt != MOE_W_INT4_G128) return MOE_ERR_UNSUPPORTED;   // bf16 token rows
    if (static_cast<long long>(s->T) * s->top_k >= (1LL << kSrcShift)) return MOE_ERR_UNSUPPORTED;
    E_loc = s->E / p->world;
    for (int r = 0; r < p->world; ++r)
        if (!p->counts[r] || !p->recv_rows[r] || !p->recv_src[r] || !p->y_ret[r] || p->pairs[r] < 0 ||
            reinterpret_cast<uintptr_t>(p->recv_rows[r]) % 16 || reinterpret_cast<uintptr_t>(p->y_ret[r]) % 16)
            return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status_t status_of(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace
}  // namespace moe

extern "C" {

moe_status_t moe_ep_count(const int32_t *offsets, const moe_shape_t *shape, const moe_ep_peers_t *peers,
                          moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_ep_count");
    int E_loc = 0;
    moe_status_t st = moe::check_ep(shape, peers, E_loc);
    if (st != MOE_OK) return st;
    const int P = shape->T * shape->top_k;
    if (!offsets && P > 0) return MOE_ERR_INVALID_ARG;
    return moe::status_of(moe::launch_pdl(moe::ep_count_kernel, dim3(1), dim3(moe::kEpThreads), 0,
                                          static_cast<cudaStream_t>(stream), offsets, P, shape->E, E_loc,
                                          peers->rank, peers->world, moe::ptrs_of(peers)));
}

moe_status_t moe_ep_dispatch(const moe_bf16_t *hidden, const int32_t *perm, const int32_t *offsets,
                             const moe_shape_t *shape, const moe_ep_peers_t *peers, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_ep_dispatch");
    int E_loc = 0;
    moe_status_t st = moe::check_ep(shape, peers, E_loc);
    if (st != MOE_OK) return st;
    const int P = shape->T * shape->top_k;
    if (P == 0) return MOE_OK;
    if (!hidden || !perm || !offsets || reinterpret_cast<uintptr_t>(hidden) % 16) return MOE_ERR_INVALID_ARG;
    const size_t smem = (3 * static_cast<size_t>(shape->E) + 1) * sizeof(int);
    return moe::status_of(moe::launch_pdl(moe::ep_dispatch_kernel, dim3(moe::ep_grid(P)), dim3(moe::kEpThreads),
                                          smem, static_cast<cudaStream_t>(stream),
                                          reinterpret_cast<const uint4 *>(hidden), perm, offsets, P, shape->top_k,
                                          shape->H / 8, shape->E, E_loc, peers->rank, peers->world, peers->capacity,
                                          moe::ptrs_of(peers), moe::device_error_flag()));
}

moe_status_t moe_ep_local_offsets(const moe_shape_t *shape, const moe_ep_peers_t *peers, int32_t *offsets_local,
                                  moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_ep_local_offsets");
    int E_loc = 0;
    moe_status_t st = moe::check_ep(shape, peers, E_loc);
    if (st != MOE_OK) return st;
    if (!offsets_local) return MOE_ERR_INVALID_ARG;
    return moe::status_of(moe::launch_pdl(moe::ep_offsets_kernel, dim3(1), dim3(moe::kEpThreads), 0,
                                          static_cast<cudaStream_t>(stream), peers->counts[peers->rank], E_loc,
                                          peers->world, offsets_local));
}

moe_status_t moe_ep_combine(const moe_bf16_t *y_local, const int32_t *offsets_local, const moe_shape_t *shape,
                            const moe_ep_peers_t *peers, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_ep_combine");
    int E_loc = 0;
    moe_status_t st = moe::check_ep(shape, peers, E_loc);
    if (st != MOE_OK) return st;
    if (!y_local || !offsets_local || reinterpret_cast<uintptr_t>(y_local) % 16) return MOE_ERR_INVALID_ARG;
    if (peers->capacity == 0) return MOE_OK;
    return moe::status_of(moe::launch_pdl(moe::ep_combine_kernel, dim3(moe::ep_grid(peers->capacity)),
                                          dim3(moe::kEpThreads), 0, static_cast<cudaStream_t>(stream),
                                          reinterpret_cast<const uint4 *>(y_local), peers->recv_src[peers->rank],
                                          offsets_local, E_loc,
                                          shape->H / 8, peers->rank, peers->world, moe::ptrs_of(peers),
                                          moe::device_error_flag()));
}

}  // extern "C"
