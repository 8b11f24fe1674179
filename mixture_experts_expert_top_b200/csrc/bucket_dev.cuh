// bucket_dev.cuh -- device building blocks of the deterministic bucketing of
// (token, expert) pairs by expert (InfiniLM PR #500 Qwen3-MoE report, §2.2
// step 1): per-warp expert histograms of contiguous pair slices, their
// prefix sums, and the stable scatter. The rank of a pair inside its expert
// comes from the histograms and __match_any_sync, never from the order of
// atomics, so the permutation is stable by pair id and deterministic.
#pragma once

#include "common.cuh"

namespace moe {

// Slice of an n-pair chunk owned by each of NW warps: a multiple of 32 pairs.
template <int NW>
__device__ __forceinline__ int warp_slice(int chunk_pairs) {
    return ((chunk_pairs + NW * 32 - 1) / (NW * 32)) * 32;
}

// hist[w*E + e] = pairs of warp w's slice routed to expert e. ids may be in
// global or shared memory. An id outside [0, E) raises kErrBadExpertId.
template <int NW>
__device__ void warp_histograms(const int32_t *ids, int begin, int n, int E, int *hist, int *err) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < NW * E; i += NW * 32) hist[i] = 0;
    __syncthreads();
    const int slice = warp_slice<NW>(n);
    for (int it = 0; it < slice; it += 32) {
        const int local = w * slice + it + lane;
        const bool in = local < n;
        const int e = in ? ids[begin + local] : -1;
        const bool ok = in && e >= 0 && e < E;
        if (in && !ok) raise_error(err, kErrBadExpertId);
        const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1);
        if (ok && lane == __ffs(m) - 1) hist[w * E + e] += __popc(m);
        __syncwarp();
    }
    __syncthreads();
}

// In place: hist[w*E+e] <- base[e] + sum_{w'<w} hist[w'*E+e].
template <int NW>
__device__ void warp_bases(int E, int *hist, const int *base) {
    for (int e = threadIdx.x; e < E; e += NW * 32) {
        int run = base[e];
        for (int w = 0; w < NW; ++w) {
            const int c = hist[w * E + e];
            hist[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
}

// Writes perm / inv_perm for the chunk, given per-warp starting rows.
template <int NW>
__device__ void warp_scatter(const int32_t *ids, int begin, int n, int E, int *hist, int32_t *__restrict__ perm,
                             int32_t *__restrict__ inv_perm) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int slice = warp_slice<NW>(n);
    const unsigned lt = (1u << lane) - 1u;
    for (int it = 0; it < slice; it += 32) {
        const int local = w * slice + it + lane;
        const bool in = local < n;
        const int e = in ? ids[begin + local] : -1;
        const bool ok = in && e >= 0 && e < E;
        const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1);
        if (ok) {
            const int r = hist[w * E + e] + __popc(m & lt);
            perm[r] = begin + local;
            inv_perm[begin + local] = r;
        } else if (in) {
            inv_perm[begin + local] = -1;
        }
        __syncwarp();
        if (ok && lane == __ffs(m) - 1) hist[w * E + e] += __popc(m);
        __syncwarp();
    }
}

// Exclusive scan of vals[0..E) into offsets[0..E] (offsets[E] = total), also
// left in shared memory `base`. A CTA of NT threads, E <= NT.
template <int NT>
__device__ void block_exclusive_scan(const int *vals, int E, int *base, int32_t *__restrict__ offsets) {
    __shared__ int warp_sums[NT / 32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int v = threadIdx.x < E ? vals[threadIdx.x] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = lane < NT / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NT / 32) warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int excl = x - v + (w > 0 ? warp_sums[w - 1] : 0);
    if (threadIdx.x < E) {
        base[threadIdx.x] = excl;
        offsets[threadIdx.x] = excl;
    }
    if (threadIdx.x == E - 1) offsets[E] = excl + v;
    __syncthreads();
}

// The whole bucketing of P pairs by one CTA of NT threads (P <= 8192).
// smem: NT/32 * E + 2 E ints.
template <int NT>
__device__ void bucket_single_cta(const int32_t *ids, int P, int E, int32_t *__restrict__ counts,
                                  int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                                  int32_t *__restrict__ inv_perm, int *smem, int *err) {
    constexpr int NW = NT / 32;
    int *hist = smem;                 // [NW * E]
    int *tot = hist + NW * E;         // [E]
    int *base = tot + E;              // [E]
    warp_histograms<NW>(ids, 0, P, E, hist, err);
    for (int e = threadIdx.x; e < E; e += NT) {
        int s = 0;
        for (int w = 0; w < NW; ++w) s += hist[w * E + e];
        tot[e] = s;
        counts[e] = s;
    }
    __syncthreads();
    block_exclusive_scan<NT>(tot, E, base, offsets);
    warp_bases<NW>(E, hist, base);
    warp_scatter<NW>(ids, 0, P, E, hist, perm, inv_perm);
}

}  // namespace moe
