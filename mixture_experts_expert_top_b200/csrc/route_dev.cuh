// route_dev.cuh -- top-k softmax routing of one token by one warp (device
// code shared by the routing kernel and the fused route + permute kernel).
//
// InfiniLM PR #500 Qwen3-MoE report, §2.1 and §2.4: each token goes to the
// top-k experts of a softmax over its router logits, and the k probabilities
// are renormalised to sum to one. Softmax is monotone, so the k largest
// probabilities are the k largest logits, and the full-softmax denominator
// cancels in the renormalisation:
//   w_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0),  l_0 = the largest logit.
// Selection compares fp32 logits only, so the ids do not depend on expf.
// Equal logits go to the lower expert id; slot order is descending logit.
#pragma once

#include <math.h>
#include <stdint.h>

namespace moe {

// Lane j of the warp ends with slot j's expert id and weight (j < k <= 32).
// Logits are read with plain loads; NaN reads as -inf.
template <int PER_LANE>
__device__ __forceinline__ void route_token(const float *row, int E, int k, int &my_id, float &my_w) {
    const int lane = threadIdx.x & 31;
    float v[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        const float x = e < E ? row[e] : -INFINITY;
        v[i] = (x != x) ? -INFINITY : x;
    }
    uint32_t taken = 0;                   // bit i: expert lane + 32 i already chosen
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i)
        if (lane + 32 * i >= E) taken |= 1u << i;

    my_id = 0;
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
    my_w = __fdiv_rn(ej, sum);
}

}  // namespace moe
