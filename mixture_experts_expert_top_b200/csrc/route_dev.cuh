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

// Order-preserving map of a logit onto uint32: larger logit, larger key.
// NaN counts as -inf and -0 as +0 (so that +0 and -0 tie, as they compare
// equal in fp32). Key 0 is below every logit and marks "not a candidate".
__device__ __forceinline__ uint32_t logit_key(float x) {
    if (x != x) x = -INFINITY;
    if (x == 0.f) x = 0.f;
    const uint32_t b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Lane j of the warp ends with slot j's expert id and weight (j < k <= 32).
// Expert e sits in lane e % 32, register e / 32. Each of the k rounds takes
// two warp reductions: the largest key left, then the lowest expert id that
// holds it; the winner's key is cleared.
template <int PER_LANE>
__device__ __forceinline__ void route_token(const float *row, int E, int k, int &my_id, float &my_w) {
    const int lane = threadIdx.x & 31;
    uint32_t key[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? logit_key(row[e]) : 0u;
    }
    my_id = 0;
    uint32_t my_key = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t local = 0;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) local = max(local, key[i]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, local);
        uint32_t cand = 0xffffffffu;
#pragma unroll
        for (int i = PER_LANE - 1; i >= 0; --i)
            if (key[i] == best) cand = static_cast<uint32_t>(lane + 32 * i);
        const int bid = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
        const bool mine = (bid & 31) == lane;
        if constexpr (PER_LANE <= 8) {
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) key[i] = (mine && i == (bid >> 5)) ? 0u : key[i];   // in registers
        } else if (mine) {
            key[bid >> 5] = 0u;
        }
        if (lane == j) {
            my_id = bid;
            my_key = best;
        }
    }
    const float l0 = key_logit(__shfl_sync(0xffffffffu, my_key, 0));
    const float ej = lane < k ? expf(key_logit(my_key) - l0) : 0.f;
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ej, j);   // slot order
    my_w = __fdiv_rn(ej, sum);
}

// Lane j >= k of a routed token takes shared slot j - k: expert E + j - k,
// weight 1 (the shared experts' outputs are added unweighted).
__device__ __forceinline__ void shared_slot(int lane, int k, int E, int &id, float &w) {
    if (lane >= k) {
        id = E + lane - k;
        w = 1.0f;
    }
}

}  // namespace moe
