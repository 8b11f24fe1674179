// permute.cu -- bucketing of the (token, expert) pairs by expert, on the GPU.
//
// InfiniLM PR #500 Qwen3-MoE report, §2.2 step 1 buckets the routing indices
// into per-expert token counts and a permutation (on the host there, behind a
// device-to-host copy, §2.3); step 2 gathers the activations by that
// permutation. Here both stay on the device:
//   counts[e]  = #{p : ids[p] = e}
//   offsets    = exclusive prefix sum of counts, offsets[E] = P
//   perm[r]    = pair id p of permuted row r; within an expert, ascending p
//   inv_perm[p] = r
// Deterministic: the rank of a pair inside its expert is computed from
// per-warp histograms in pair order, never from the order of atomics.
//
// Layout of the work: a CTA owns a chunk of consecutive pairs; warp w owns a
// contiguous slice of the chunk and walks it 32 pairs at a time, using
// __match_any_sync to rank equal experts inside each step. One CTA of 1024
// threads does everything when P <= kSingleMax; otherwise three kernels run:
// per-chunk histograms (CTAs of 512 threads, kChunk pairs each), one scan CTA,
// per-chunk scatter.
#include "bucket_dev.cuh"
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;        // single-CTA path and the scan CTA
constexpr int kSingleMax = 8192;      // pairs handled by the single-CTA path
constexpr int kChunkThreads = 512;    // multi-CTA path
constexpr int kChunk = 2048;          // pairs per CTA on the multi-CTA path

// All pairs in one CTA.
__global__ void __launch_bounds__(kThreads, 1)
permute_single_kernel(const int32_t *__restrict__ ids, int P, int E, int32_t *__restrict__ counts,
                      int32_t *__restrict__ offsets, int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm,
                      int *err) {
    extern __shared__ int smem[];
    griddep_launch_dependents();
    griddep_wait();
    bucket_single_cta<kThreads>(ids, P, E, counts, offsets, perm, inv_perm, smem, err);
}

// Multi-CTA pass 1: chunk_hist[c*E + e].
__global__ void __launch_bounds__(kChunkThreads)
permute_count_kernel(const int32_t *__restrict__ ids, int P, int E, int32_t *__restrict__ chunk_hist, int *err) {
    constexpr int NW = kChunkThreads / 32;
    extern __shared__ int smem[];
    griddep_launch_dependents();
    griddep_wait();
    const int begin = blockIdx.x * kChunk;
    const int n = min(kChunk, P - begin);
    warp_histograms<NW>(ids, begin, n, E, smem, err);
    for (int e = threadIdx.x; e < E; e += kChunkThreads) {
        int s = 0;
        for (int w = 0; w < NW; ++w) s += smem[w * E + e];
        chunk_hist[static_cast<size_t>(blockIdx.x) * E + e] = s;
    }
}

// Multi-CTA pass 2 (one CTA): counts, offsets, and chunk_hist turned into the
// first row of each (chunk, expert). G = kThreads / E threads (a power of two,
// at most 32, so one warp segment) share an expert: thread `part` owns a
// contiguous run of chunks. Loads go out 8 at a time, so the walk over the
// chunks is not one L2 round trip per chunk.
__global__ void __launch_bounds__(kThreads, 1)
permute_scan_kernel(int nchunks, int E, int32_t *__restrict__ chunk_hist, int32_t *__restrict__ counts,
                    int32_t *__restrict__ offsets) {
    extern __shared__ int smem[];
    griddep_launch_dependents();
    griddep_wait();
    int *tot = smem;        // [E]
    int *base = tot + E;    // [E]
    int G = 1;
    while (G < 32 && 2 * G * E <= kThreads) G *= 2;
    const int e = threadIdx.x / G, part = threadIdx.x % G;
    const bool active = e < E;
    const int per = (nchunks + G - 1) / G;
    const int c0 = part * per, c1 = min(nchunks, c0 + per);
    int sum = 0;
    if (active) {
        for (int c = c0; c < c1; c += 8) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = c + j < c1 ? __ldcg(chunk_hist + static_cast<size_t>(c + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) sum += v[j];
        }
    }
    // exclusive scan of `sum` over the G threads of this expert (lanes of one segment)
    const int lane = threadIdx.x & 31;
    int incl = sum;
    for (int o = 1; o < G; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if ((lane % G) >= o) incl += y;
    }
    const int seg_last = (lane / G) * G + G - 1;
    const int total = __shfl_sync(0xffffffffu, incl, seg_last);
    if (active && part == 0) {
        tot[e] = total;
        counts[e] = total;
    }
    __syncthreads();
    block_exclusive_scan<kThreads>(tot, E, base, offsets);
    if (active) {
        int run = base[e] + incl - sum;
        for (int c = c0; c < c1; c += 8) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = c + j < c1 ? __ldcg(chunk_hist + static_cast<size_t>(c + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (c + j < c1) {
                    chunk_hist[static_cast<size_t>(c + j) * E + e] = run;
                    run += v[j];
                }
        }
    }
}

// Multi-CTA passes 2 and 3 in one kernel, for few chunks (E <= the CTA's
// threads): every CTA derives its chunk's first rows from all the chunk
// counts itself (nchunks * E ints from L2), so neither the scan CTA nor its
// launch is needed. G threads share an expert, as in permute_scan_kernel.
// CTA 0 also writes counts and offsets.
constexpr int kFusedScanMaxChunks = 64;

__global__ void __launch_bounds__(kChunkThreads)
permute_scan_scatter_kernel(const int32_t *__restrict__ ids, int P, int E, int nchunks,
                            const int32_t *__restrict__ chunk_hist, int32_t *__restrict__ counts,
                            int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                            int32_t *__restrict__ inv_perm) {
    constexpr int NW = kChunkThreads / 32;
    extern __shared__ int smem[];
    int *hist = smem;                 // [NW * E]
    int *tot = hist + NW * E;         // [E] rows of expert e
    int *base = tot + E;              // [E] first row of expert e, then of this chunk's rows of e
    int *before = base + E;           // [E] rows of expert e in the chunks before this one
    int *offs_local = before + E;     // [E + 1] where CTAs other than 0 put the offsets
    griddep_launch_dependents();
    griddep_wait();
    int G = 1;
    while (G < 32 && 2 * G * E <= kChunkThreads) G *= 2;
    const int e = threadIdx.x / G, part = threadIdx.x % G;
    const bool active = e < E;
    const int per = (nchunks + G - 1) / G;
    const int c0 = part * per, c1 = min(nchunks, c0 + per);
    const int me = static_cast<int>(blockIdx.x);
    int sum = 0, pre = 0;
    if (active) {
        for (int c = c0; c < c1; c += 8) {
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = c + j < c1 ? __ldcg(chunk_hist + static_cast<size_t>(c + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sum += v[j];
                if (c + j < me) pre += v[j];
            }
        }
    }
    for (int o = G / 2; o > 0; o >>= 1) {      // over the G lanes of the expert (an aligned lane segment)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        pre += __shfl_xor_sync(0xffffffffu, pre, o);
    }
    if (active && part == 0) {
        tot[e] = sum;
        before[e] = pre;
        if (me == 0) counts[e] = sum;
    }
    __syncthreads();
    block_exclusive_scan<kChunkThreads>(tot, E, base, me == 0 ? offsets : offs_local);
    for (int i = threadIdx.x; i < E; i += kChunkThreads) base[i] += before[i];
    const int begin = me * kChunk;
    const int n = min(kChunk, P - begin);
    warp_histograms<NW>(ids, begin, n, E, hist, nullptr);   // its first barrier also orders base
    warp_bases<NW>(E, hist, base);
    warp_scatter<NW>(ids, begin, n, E, hist, perm, inv_perm);
}

// Multi-CTA pass 3: scatter each chunk from its per-expert first rows.
__global__ void __launch_bounds__(kChunkThreads)
permute_scatter_kernel(const int32_t *__restrict__ ids, int P, int E, const int32_t *__restrict__ chunk_base,
                       int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm) {
    constexpr int NW = kChunkThreads / 32;
    extern __shared__ int smem[];
    int *hist = smem;                 // [NW * E]
    int *base = hist + NW * E;        // [E]
    griddep_launch_dependents();
    griddep_wait();
    const int begin = blockIdx.x * kChunk;
    const int n = min(kChunk, P - begin);
    for (int e = threadIdx.x; e < E; e += kChunkThreads)
        base[e] = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
    warp_histograms<NW>(ids, begin, n, E, hist, nullptr);
    warp_bases<NW>(E, hist, base);
    warp_scatter<NW>(ids, begin, n, E, hist, perm, inv_perm);
}

// hidden_perm[r] = hidden[perm[r] / k]: one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ perm, int P, int vecs_per_row,
                   int k, uint4 *__restrict__ out, int *err) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < P; r += warps) {
        int p = __ldg(perm + r);
        if (kDebugBounds && (p < 0 || p >= P)) {
            raise_error(err, kErrBounds);
            p = 0;
        }
        const uint4 *src = hidden + static_cast<size_t>(p / k) * vecs_per_row;
        uint4 *dst = out + static_cast<size_t>(r) * vecs_per_row;
        // all loads of a 4 KB slice are in flight before its stores; the copy is
        // written once and read once by the next kernel: stream it past L2 so
        // that the k-times-reused hidden rows stay resident
        for (int v0 = 0; v0 < vecs_per_row; v0 += 32 * 8) {
            uint4 buf[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int v = v0 + 32 * j + lane;
                if (v < vecs_per_row) buf[j] = __ldg(src + v);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int v = v0 + 32 * j + lane;
                if (v < vecs_per_row) __stcs(dst + v, buf[j]);
            }
        }
    }
}

}  // namespace

int permute_kernel_count(long long P, int E) {
    if (P <= kSingleMax) return 1;
    const long long nchunks = (P + kChunk - 1) / kChunk;
    return nchunks <= kFusedScanMaxChunks && E <= kChunkThreads ? 2 : 3;
}

size_t permute_scratch_bytes(long long P, int E) {
    if (P <= kSingleMax) return 0;
    const long long nchunks = (P + kChunk - 1) / kChunk;
    return static_cast<size_t>(nchunks) * E * sizeof(int32_t);
}

cudaError_t launch_permute(const int32_t *ids, int P, int E, int32_t *counts, int32_t *offsets, int32_t *perm,
                           int32_t *inv_perm, void *scratch, int *err, cudaStream_t s) {
    cudaError_t st;
    if (P <= kSingleMax) {
        const size_t sm = (static_cast<size_t>(kThreads / 32) * E + 2 * E) * sizeof(int);
        st = ensure_dynamic_smem(permute_single_kernel, sm);
        if (st != cudaSuccess) return st;
        return launch_pdl(permute_single_kernel, dim3(1), dim3(kThreads), sm, s, ids, P, E, counts, offsets, perm,
                          inv_perm, err);
    }
    const int nchunks = (P + kChunk - 1) / kChunk;
    int32_t *chunk_hist = static_cast<int32_t *>(scratch);
    const size_t sm_hist = static_cast<size_t>(kChunkThreads / 32) * E * sizeof(int);
    const size_t sm_scatter = (static_cast<size_t>(kChunkThreads / 32) * E + E) * sizeof(int);
    st = ensure_dynamic_smem(permute_count_kernel, sm_hist);
    if (st != cudaSuccess) return st;
    st = ensure_dynamic_smem(permute_scatter_kernel, sm_scatter);
    if (st != cudaSuccess) return st;
    if ((st = launch_pdl(permute_count_kernel, dim3(nchunks), dim3(kChunkThreads), sm_hist, s, ids, P, E, chunk_hist,
                         err)) != cudaSuccess)
        return st;
    if (permute_kernel_count(P, E) == 2) {
        const size_t sm_fused = (static_cast<size_t>(kChunkThreads / 32) * E + 4 * E + 1) * sizeof(int);
        if ((st = ensure_dynamic_smem(permute_scan_scatter_kernel, sm_fused)) != cudaSuccess) return st;
        return launch_pdl(permute_scan_scatter_kernel, dim3(nchunks), dim3(kChunkThreads), sm_fused, s, ids, P, E,
                          nchunks, static_cast<const int32_t *>(chunk_hist), counts, offsets, perm, inv_perm);
    }
    if ((st = launch_pdl(permute_scan_kernel, dim3(1), dim3(kThreads), 2 * E * sizeof(int), s, nchunks, E,
                         chunk_hist, counts, offsets)) != cudaSuccess)
        return st;
    return launch_pdl(permute_scatter_kernel, dim3(nchunks), dim3(kChunkThreads), sm_scatter, s, ids, P, E,
                      static_cast<const int32_t *>(chunk_hist), perm, inv_perm);
}

cudaError_t launch_gather(const uint16_t *hidden, const int32_t *perm, int P, int H, int k, uint16_t *hidden_perm,
                          int *err, cudaStream_t s) {
    if (P == 0) return cudaSuccess;
    const int rows_per_block = 8;
    int blocks = (P + rows_per_block - 1) / rows_per_block;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(32 * rows_per_block), 0, s,
                      reinterpret_cast<const uint4 *>(hidden), perm, P, H / 8, k, reinterpret_cast<uint4 *>(hidden_perm),
                      err);
}

}  // namespace moe
