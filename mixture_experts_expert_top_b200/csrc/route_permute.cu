// route_permute.cu -- routing and bucketing of a small batch in one CTA.
//
// InfiniLM PR #500 Qwen3-MoE report, §2.1 (top-k softmax routing with
// renormalisation) followed by §2.2 step 1 (bucketing of the (token, expert)
// pairs by expert). For a decode batch both steps are tiny and the cost is
// the launch and the round trip of the ids through global memory, so one CTA
// of 1024 threads does both: 32 warps route the tokens (one token per warp at
// a time, route_token of route_dev.cuh), the ids stay in shared memory, and
// the same CTA buckets them (bucket_single_cta of bucket_dev.cuh). The outputs
// are bit-identical to launch_route followed by launch_permute.
#include "bucket_dev.cuh"
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;
constexpr int kMaxTokens = 64;      // at most 2 tokens per warp: each token is latency-bound
constexpr int kMaxPairs = 8192;
constexpr int kMaxExperts = 256;    // at most 8 logits per lane

template <int PER_LANE>
__global__ void __launch_bounds__(kThreads, 1)
route_permute_kernel(const float *__restrict__ logits, int T, int E, int k, int n_shared, int32_t *__restrict__ ids,
                     float *__restrict__ w, int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                     int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm, int *err) {
    // E routed experts and k routed slots; the bucketing sees E + n_shared
    // experts and K = k + n_shared slots per token
    const int K = k + n_shared, Et = E + n_shared;
    extern __shared__ int smem[];
    int *bucket_smem = smem;                                   // [(32 + 2) * Et]
    int32_t *ids_s = smem + (kThreads / 32 + 2) * Et;          // [T * K]
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    for (int t = threadIdx.x >> 5; t < T; t += kThreads / 32) {
        int id;
        float wt;
        route_token<PER_LANE>(logits + static_cast<size_t>(t) * E, E, k, id, wt);
        shared_slot(lane, k, E, id, wt);
        if (lane < K) {
            ids[static_cast<size_t>(t) * K + lane] = id;
            w[static_cast<size_t>(t) * K + lane] = wt;
            ids_s[t * K + lane] = id;
        }
    }
    __syncthreads();
    bucket_single_cta<kThreads>(ids_s, T * K, Et, counts, offsets, perm, inv_perm, bucket_smem, err);
}

template <int PER_LANE>
cudaError_t launch_t(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w, int32_t *counts,
                     int32_t *offsets, int32_t *perm, int32_t *inv_perm, int *err, cudaStream_t s) {
    const int K = k + n_shared, Et = E + n_shared;
    const size_t sm = (static_cast<size_t>(kThreads / 32 + 2) * Et + static_cast<size_t>(T) * K) * sizeof(int);
    const cudaError_t st = ensure_dynamic_smem(route_permute_kernel<PER_LANE>, sm);
    if (st != cudaSuccess) return st;
    return launch_pdl(route_permute_kernel<PER_LANE>, dim3(1), dim3(kThreads), sm, s, logits, T, E, k, n_shared,
                      ids, w, counts, offsets, perm, inv_perm, err);
}

}  // namespace

bool route_permute_fusable(int T, int E, int k) {
    return T > 0 && T <= kMaxTokens && static_cast<long long>(T) * k <= kMaxPairs && E <= kMaxExperts;
}

cudaError_t launch_route_permute(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w,
                                 int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm, int *err,
                                 cudaStream_t s) {
    if (!route_permute_fusable(T, E + n_shared, k + n_shared)) return cudaErrorInvalidValue;
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 1) return launch_t<1>(logits, T, E, k, n_shared, ids, w, counts, offsets, perm, inv_perm, err, s);
    if (per_lane <= 2) return launch_t<2>(logits, T, E, k, n_shared, ids, w, counts, offsets, perm, inv_perm, err, s);
    if (per_lane <= 4) return launch_t<4>(logits, T, E, k, n_shared, ids, w, counts, offsets, perm, inv_perm, err, s);
    return launch_t<8>(logits, T, E, k, n_shared, ids, w, counts, offsets, perm, inv_perm, err, s);
}

}  // namespace moe
