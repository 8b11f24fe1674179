// route.cu -- top-k softmax routing with renormalisation, one warp per token
// (the per-token logic is route_token in route_dev.cuh).
//
// InfiniLM PR #500 Qwen3-MoE report, §2.1 and §2.4: Qwen3-MoE routes each
// token to the top-k experts of a softmax over the router logits (no bias,
// no shared expert); the k probabilities are renormalised to sum to one.
// Because softmax is monotone, the k largest probabilities are the k largest
// logits, and the full-softmax denominator cancels in the renormalisation:
//   w_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0),  l_0 = the largest logit.
// Selection compares fp32 logits only, so the ids do not depend on expf.
// Equal logits go to the lower expert id; slot order is descending logit.
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 4;

template <int PER_LANE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
route_kernel(const float *__restrict__ logits, int T, int E, int k, int n_shared, int32_t *__restrict__ ids,
             float *__restrict__ w) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (t >= T) return;
    int id;
    float wt;
    route_token<PER_LANE>(logits + static_cast<size_t>(t) * E, E, k, id, wt);
    // routed slots 0..k-1, then the shared experts E.. with weight 1
    shared_slot(lane, k, E, id, wt);
    const int K = k + n_shared;
    if (lane < K) {
        ids[static_cast<size_t>(t) * K + lane] = id;
        w[static_cast<size_t>(t) * K + lane] = wt;
    }
}

template <int PER_LANE>
cudaError_t launch_route_t(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w,
                           cudaStream_t s) {
    const int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    return launch_pdl(route_kernel<PER_LANE>, dim3(blocks), dim3(kWarpsPerBlock * 32), 0, s, logits, T, E, k,
                      n_shared, ids, w);
}

}  // namespace

cudaError_t launch_route(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w,
                         cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 1) return launch_route_t<1>(logits, T, E, k, n_shared, ids, w, s);
    if (per_lane <= 2) return launch_route_t<2>(logits, T, E, k, n_shared, ids, w, s);
    if (per_lane <= 4) return launch_route_t<4>(logits, T, E, k, n_shared, ids, w, s);
    if (per_lane <= 8) return launch_route_t<8>(logits, T, E, k, n_shared, ids, w, s);
    if (per_lane <= 16) return launch_route_t<16>(logits, T, E, k, n_shared, ids, w, s);
    return launch_route_t<32>(logits, T, E, k, n_shared, ids, w, s);
}

}  // namespace moe
