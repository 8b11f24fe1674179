// route.cu -- top-k softmax routing with renormalisation, one warp per token.
//
// InfiniLM PR #500 Qwen3-MoE report, §2.1 and §2.4: Qwen3-MoE routes each
// token to the top-k experts of a softmax over the router logits (no bias,
// no shared expert); the k probabilities are renormalised to sum to one.
// Because softmax is monotone, the k largest probabilities are the k largest
// logits, and the full-softmax denominator cancels in the renormalisation:
//   w_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0),  l_0 = the largest logit.
// Selection compares fp32 logits only, so the ids do not depend on expf.
// Equal logits go to the lower expert id; slot order is descending logit.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 4;
constexpr int kMaxPerLane = 32;   // E <= 1024

template <int PER_LANE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
route_kernel(const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ ids,
             float *__restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *row = logits + static_cast<size_t>(t) * E;

    float v[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        float x = e < E ? __ldg(row + e) : -INFINITY;
        v[i] = (x != x) ? -INFINITY : x;   // NaN reads as -inf
    }
    uint32_t taken = 0;                   // bit i: expert lane + 32 i already chosen
    for (int i = 0; i < PER_LANE; ++i)
        if (lane + 32 * i >= E) taken |= 1u << i;

    int my_id = 0;          // lane j keeps slot j
    float my_logit = 0.f;
    for (int j = 0; j < k; ++j) {
        float best = -INFINITY;
        int bid = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            const int e = lane + 32 * i;
            if (!((taken >> i) & 1u) && (v[i] > best || (v[i] == best && e < bid))) {
                best = v[i];
                bid = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bid, o);
            if (ob > best || (ob == best && oi < bid)) {
                best = ob;
                bid = oi;
            }
        }
        if ((bid & 31) == lane) taken |= 1u << (bid >> 5);
        if (lane == j) {
            my_id = bid;
            my_logit = best;
        }
    }

    const float l0 = __shfl_sync(0xffffffffu, my_logit, 0);
    const float ej = lane < k ? expf(my_logit - l0) : 0.f;
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ej, j);   // slot order
    if (lane < k) {
        ids[static_cast<size_t>(t) * k + lane] = my_id;
        w[static_cast<size_t>(t) * k + lane] = __fdiv_rn(ej, sum);
    }
}

template <int PER_LANE>
cudaError_t launch_route_t(const float *logits, int T, int E, int k, int32_t *ids, float *w, cudaStream_t s) {
    const int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    route_kernel<PER_LANE><<<blocks, kWarpsPerBlock * 32, 0, s>>>(logits, T, E, k, ids, w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *ids, float *w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 1) return launch_route_t<1>(logits, T, E, k, ids, w, s);
    if (per_lane <= 2) return launch_route_t<2>(logits, T, E, k, ids, w, s);
    if (per_lane <= 4) return launch_route_t<4>(logits, T, E, k, ids, w, s);
    if (per_lane <= 8) return launch_route_t<8>(logits, T, E, k, ids, w, s);
    if (per_lane <= 16) return launch_route_t<16>(logits, T, E, k, ids, w, s);
    return launch_route_t<kMaxPerLane>(logits, T, E, k, ids, w, s);
}

}  // namespace moe
