// finalize.cu -- weighted combine of the k expert outputs of each token.
//
// FlashInfer PR #7196 analysis, §1 (moe_finalize.py / moe_unpermute): the
// first slot is a round-to-nearest fp32 multiply (so the sign of a zero
// product survives), every later slot a round-to-nearest fp32 FMA in slot
// order, and no flush-to-zero anywhere (the PR removed .ftz), so subnormal
// partial sums survive:
//   acc = v_0 * w_0;  acc = fma(v_j, w_j, acc), j = 1..k-1;  out = bf16_rne(acc)
// The gather-combine reads the k rows of y through inv_perm, so no atomics
// and no scatter are involved: the result is deterministic.
//
// Memory layout of the work: one thread owns 8 consecutive hidden elements
// (one 16-byte vector) of one token; a warp reads 512 contiguous bytes of each
// y row it touches. HBM-bound: (k*H + H)*2 bytes + k*(4+4) bytes per token.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2_rne(float lo, float hi) {
    const __nv_bfloat16 a = __float2bfloat16_rn(lo);
    const __nv_bfloat16 b = __float2bfloat16_rn(hi);
    return static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

__global__ void __launch_bounds__(256)
finalize_kernel(const uint4 *__restrict__ y, const float *__restrict__ w, const int32_t *__restrict__ inv_perm,
                int T, int vecs_per_row, int k, int P, uint4 *__restrict__ out) {
    const long long total = static_cast<long long>(T) * vecs_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / vecs_per_row);
        const int v = static_cast<int>(i - static_cast<long long>(t) * vecs_per_row);
        float acc[8];
        for (int j = 0; j < k; ++j) {
            const int r = __ldg(inv_perm + static_cast<size_t>(t) * k + j);
            const float wj = __ldg(w + static_cast<size_t>(t) * k + j);
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            if (r >= 0 && r < P) q = __ldg(y + static_cast<size_t>(r) * vecs_per_row + v);
            const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = bf16_bits_to_float((qs[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                acc[e] = (j == 0) ? __fmul_rn(x, wj) : __fmaf_rn(x, wj, acc[e]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2_rne(acc[0], acc[1]);
        o.y = pack_bf16x2_rne(acc[2], acc[3]);
        o.z = pack_bf16x2_rne(acc[4], acc[5]);
        o.w = pack_bf16x2_rne(acc[6], acc[7]);
        out[i] = o;
    }
}

}  // namespace

cudaError_t launch_finalize(const uint16_t *y, const float *w, const int32_t *inv_perm, int T, int H, int k,
                            uint16_t *out, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int vpr = H / 8;
    const long long total = static_cast<long long>(T) * vpr;
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    finalize_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(reinterpret_cast<const uint4 *>(y), w, inv_perm, T,
                                                             vpr, k, T * k, reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace moe
