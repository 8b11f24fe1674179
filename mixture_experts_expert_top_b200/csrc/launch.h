// launch.h -- host-side launchers of the libmoe_b200 kernels. Internal to the
// library: the C ABI in include/moe.h validates arguments and calls these.
// Every launcher enqueues on `stream` and returns the cudaGetLastError() of
// its launches.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"
#include "nvtx3/nvToolsExt.h"

namespace moe {

// An NVTX range named after a C-ABI entry point, open for the host-side
// duration of the call (argument checks and enqueueing). Costs a predicted
// branch when no profiler has attached an NVTX tool.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// ---- capi.cu
// The shape rules every entry point applies (MOE_OK or the status to return).
moe_status_t validate_shape(const moe_shape_t *shape);
// Slots per token (top_k routed + n_shared shared) and experts in the weight
// arrays (E routed + n_shared shared): what permute, the GEMMs and finalize see.
int shape_slots(const moe_shape_t *shape);
int shape_experts(const moe_shape_t *shape);
// Device address of the library's error flag word on the current device.
int *device_error_flag();

// ---- selftest.cu
// One CTA waits limit_ns on an mbarrier that nothing arrives on (the
// bounded-wait path: the wait gives up and raises the timeout code).
cudaError_t launch_bounded_wait_selftest(unsigned long long limit_ns, int *err, cudaStream_t s);

// ---- route.cu
// ids/w rows hold k routed slots, then n_shared slots of experts E.. with
// weight 1 (row stride k + n_shared).
cudaError_t launch_route(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w,
                         cudaStream_t s);

// ---- route_permute.cu
// Routing and bucketing of a small batch by one CTA (same outputs as
// launch_route followed by launch_permute).
// E and k here count all experts and slots (shared included).
bool route_permute_fusable(int T, int E, int k);
// E routed experts, k routed slots, n_shared shared experts / slots.
cudaError_t launch_route_permute(const float *logits, int T, int E, int k, int n_shared, int32_t *ids, float *w,
                                 int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm, int *err,
                                 cudaStream_t s);

// ---- permute.cu
// Scratch bytes the permute needs for P pairs over E experts (0 when a
// single CTA handles all pairs).
size_t permute_scratch_bytes(long long P, int E);
// Kernels launch_permute enqueues for P pairs over E experts (1, 2 or 3).
int permute_kernel_count(long long P, int E);
cudaError_t launch_permute(const int32_t *ids, int P, int E, int32_t *counts, int32_t *offsets, int32_t *perm,
                           int32_t *inv_perm, void *scratch, int *err, cudaStream_t s);
cudaError_t launch_gather(const uint16_t *hidden, const int32_t *perm, int P, int H, int k, uint16_t *hidden_perm,
                          int *err, cudaStream_t s);

// ---- finalize.cu
cudaError_t launch_finalize(const uint16_t *y, const float *w, const int32_t *inv_perm, int T, int H, int k,
                            uint16_t *out, int *err, cudaStream_t s);

// ---- gemm_sm100.cu
struct GemmArgs {
    const void *a;              // activations [P, K] bf16 in permuted row order, or, when perm is
                                // given, hidden [T, K] with row r of the operand = a[perm[r] / top_k]
    const int32_t *perm;        // optional [P]: gather the token operand through it
    int T, top_k;               // rows of `a` and pairs per token (used with perm)
    const int32_t *offsets;     // [E+1]
    const void *w;              // weights (bf16 [E, rows, K] or int4 [E, rows, K/2])
    const uint16_t *w_scales;   // int4 only: [E, rows, K/128] bf16
    int P, E, K;
    int m_out;                  // output features: I (gate/up) or H (down)
    int w_rows;                 // weight rows per expert: 2I or H
    int fmt;                    // 0 bf16, 1 int4 g128
    bool swiglu;
    uint16_t *out;              // [P, m_out] bf16
    int *err;
    int hints = 0;              // kGemmHint* bits, set only by moe_forward
};
// The kernel before this GEMM on the stream started after `offsets` was
// complete, so the GEMM may read offsets and load weight tiles before
// griddepcontrol.wait (only the token operand depends on the kernel before).
constexpr int kGemmHintOffsetsReady = 1;
// Before griddepcontrol.wait, prefetch into L2 the weights of the tile this
// CTA would get if every expert had one token block (a guess: a wrong one
// costs only bandwidth).
constexpr int kGemmHintPrefetchGuess = 2;
cudaError_t launch_grouped_gemm(const GemmArgs &g, cudaStream_t s);
// True when the gate/up GEMM for this shape should read the token rows through
// perm itself (few rows per expert) rather than from a gathered copy.
bool gemm_gathers_in_kernel(int P, int E, int fmt);
// ---- gemm_prefill_sm100.cu: bf16, tokens on the MMA's M side (many tokens per expert)
cudaError_t launch_grouped_gemm_prefill(const GemmArgs &g, cudaStream_t s);
// ---- gemm_wm_pair_sm100.cu: bf16, weights on M across a CTA pair (M = 256),
// tokens on N with N = the tile's rows rounded up to 16 (permuted rows, no perm)
cudaError_t launch_grouped_gemm_wm_pair(const GemmArgs &g, cudaStream_t s);
cudaError_t launch_dequant_int4(const uint8_t *q, const uint16_t *scales, int rows, int K, uint16_t *out,
                                cudaStream_t s);
// ---- gemm_int4_warp_sm100.cu: the W4A16 down GEMM for few rows per expert
// (P/E <= 24): int4 decoded in registers straight into warp-level MMA
// fragments (swiglu must be false)
cudaError_t launch_grouped_gemm_int4_warp(const GemmArgs &g, cudaStream_t s);

// ---- gemm_mxfp8_sm100.cu: MXFP8 weights (E4M3 + one E8M0 scale per 32 K),
// block-scaled tcgen05 MMA; the token operand is MX-quantised too.
struct MxGemmArgs {
    GemmArgs base;              // base.a: token rows as E4M3 bytes; base.out: y (down) as bf16
    const uint8_t *w_sf;        // [E * w_rows, K/32] E8M0 weight scales
    const uint8_t *x_sf;        // [rows of base.a, K/32] E8M0 token scales
    uint8_t *out_q;             // gate/up: act E4M3 [P, I]
    uint8_t *out_sf;            // gate/up: act E8M0 [P, I/32]
};
cudaError_t launch_grouped_gemm_mxfp8(const MxGemmArgs &g, cudaStream_t s);
// ---- fused_decode_sm100.cu: the whole bf16 layer for a decode batch in one
// persistent kernel (T <= 64, k + S <= 16, E + S <= 256). done:
// fused_counter_words(E, S) counters of the workspace, zeroed on the stream
// by the launcher before the kernel.
size_t fused_counter_words(int E, int S);
bool fused_decode_supported(int T, int H, int I, int E, int k, int S, int fmt);
cudaError_t launch_fused_decode(const float *logits, const uint16_t *hidden, const void *w_gu, const void *w_d,
                                int T, int H, int I, int E, int k, int S, int32_t *ids, float *w, int32_t *counts,
                                int32_t *offsets, int32_t *perm, int32_t *inv_perm, uint16_t *act, uint16_t *y,
                                uint16_t *out, unsigned int *done, int *err, cudaStream_t s);
// bf16 rows [rows, K] -> E4M3 [rows, K] and E8M0 [rows, K/32] (K % 32 == 0).
cudaError_t launch_mx_quantize(const uint16_t *x, int rows, int K, uint8_t *q, uint8_t *scales, cudaStream_t s);

}  // namespace moe
