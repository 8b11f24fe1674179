// finalize.cu -- weighted combine of the k expert outputs of each token.
//
// FlashInfer PR #7196 analysis, §1 (moe_finalize.py / moe_unpermute): the
// first slot is a round-to-nearest fp32 multiply (so the sign of a zero
// product survives), every later slot a round-to-nearest fp32 FMA in slot
// order, and no flush-to-zero anywhere (the PR removed .ftz), so subnormal
// partial sums survive:
//   acc = v_0 * w_0;  acc = fma(v_j, w_j, acc), j = 1..k-1;  out = bf16_rne(acc)
// The gather-combine reads the k rows of y through inv_perm, so no atomics
// and no scatter are involved: the result is deterministic. A row index
// outside [0, T*k) contributes 0 and raises kErrBadRow on the device flag.
//
// Memory layout of the work: one thread owns 8 consecutive hidden elements
// (one 16-byte vector) of one token; a warp reads 512 contiguous bytes of each
// y row it touches. HBM-bound: (k*H + H)*2 bytes + k*(4+4) bytes per token.
#include "common.cuh"
#include "launch.h"
#include "launch_util.cuh"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2_rne(float lo, float hi) {
    const __nv_bfloat16 a = __float2bfloat16_rn(lo);
    const __nv_bfloat16 b = __float2bfloat16_rn(hi);
    return static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// KT > 0: top_k known at compile time, so the k row indices, weights and
// 16-byte row loads of a thread are all issued before the combine.
template <int KT>
__global__ void __launch_bounds__(256)
finalize_kernel(const uint4 *__restrict__ y, const float *__restrict__ w, const int32_t *__restrict__ inv_perm,
                int T, int vecs_per_row, int k_rt, int P, uint4 *__restrict__ out, int *err) {
    griddep_wait();     // no early trigger: the next kernel's CTAs would share SMs with this one
    const int k = KT > 0 ? KT : k_rt;
    const long long total = static_cast<long long>(T) * vecs_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / vecs_per_row);
        const int v = static_cast<int>(i - static_cast<long long>(t) * vecs_per_row);
        float acc[8];
        if constexpr (KT > 0) {
            int r[KT];
            float wj[KT];
            uint4 q[KT];
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                r[j] = __ldg(inv_perm + static_cast<size_t>(t) * KT + j);
                wj[j] = __ldg(w + static_cast<size_t>(t) * KT + j);
            }
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                const bool ok = r[j] >= 0 && r[j] < P;
                if (!ok && v == 0) raise_error(err, kErrBadRow);
                q[j] = ok ? __ldcs(y + static_cast<size_t>(r[j]) * vecs_per_row + v)
                          : make_uint4(0u, 0u, 0u, 0u);   // y is read once
            }
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                const uint32_t qs[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = bf16_bits_to_float((qs[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                    acc[e] = (j == 0) ? __fmul_rn(x, wj[j]) : __fmaf_rn(x, wj[j], acc[e]);
                }
            }
        } else {
            for (int j = 0; j < k; ++j) {
                const int r = __ldg(inv_perm + static_cast<size_t>(t) * k + j);
                const float wj = __ldg(w + static_cast<size_t>(t) * k + j);
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (r >= 0 && r < P)
                    q = __ldg(y + static_cast<size_t>(r) * vecs_per_row + v);
                else if (v == 0)
                    raise_error(err, kErrBadRow);
                const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = bf16_bits_to_float((qs[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                    acc[e] = (j == 0) ? __fmul_rn(x, wj) : __fmaf_rn(x, wj, acc[e]);
                }
            }
        }
        uint4 o;
        o.x = pack_bf16x2_rne(acc[0], acc[1]);
        o.y = pack_bf16x2_rne(acc[2], acc[3]);
        o.z = pack_bf16x2_rne(acc[4], acc[5]);
        o.w = pack_bf16x2_rne(acc[6], acc[7]);
        __stcs(out + i, o);
    }
}

template <int KT>
cudaError_t launch_finalize_t(int blocks, cudaStream_t s, const uint16_t *y, const float *w, const int32_t *inv_perm,
                              int T, int vpr, int k, int P, uint16_t *out, int *err) {
    return launch_pdl(finalize_kernel<KT>, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4 *>(y), w,
                      inv_perm, T, vpr, k, P, reinterpret_cast<uint4 *>(out), err);
}

}  // namespace

cudaError_t launch_finalize(const uint16_t *y, const float *w, const int32_t *inv_perm, int T, int H, int k,
                            uint16_t *out, int *err, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int vpr = H / 8;
    const long long total = static_cast<long long>(T) * vpr;
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    const int b = static_cast<int>(blocks);
    switch (k) {
        case 1: return launch_finalize_t<1>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
        case 2: return launch_finalize_t<2>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
        case 4: return launch_finalize_t<4>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
        case 6: return launch_finalize_t<6>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
        case 8: return launch_finalize_t<8>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
        default: return launch_finalize_t<0>(b, s, y, w, inv_perm, T, vpr, k, T * k, out, err);
    }
}

}  // namespace moe
