/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE expert-FFN layer library,
 * libmoe_b200.so.
 *
 * The layer (InfiniLM PR #500 Qwen3-MoE report, §2.2; FlashInfer PR #7196
 * analysis, §1-§2):
 *
 *   route     top-k of a softmax over E router logits, renormalised over k
 *   permute   bucket the T*k (token, expert) pairs by expert: counts, offsets,
 *             a stable permutation, and optionally the gathered activations
 *   gate/up   per expert, act = bf16(silu(x W_g^T) * (x W_u^T)), fp32 accumulate
 *   down      per expert, y = bf16(act W_d^T), fp32 accumulate
 *   finalize  out[t] = bf16(w_0 v_0 (+) w_1 v_1 (+) ...), slot order, fp32
 *
 * Conventions (all entry points):
 *  - Every buffer argument is a DEVICE pointer unless its name ends in
 *    "_host". The caller allocates and frees every buffer; the library never
 *    allocates device or host memory on these paths.
 *  - Row-major, contiguous. bf16 values are passed as their 16-bit patterns
 *    (moe_bf16_t). Index arrays are int32.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and is asynchronous unless stated otherwise.
 *  - Arguments are validated before anything is enqueued; a non-OK status
 *    means nothing was launched. T = 0 is valid and enqueues nothing.
 *  - Shape limits: 1 <= E <= 1024, 1 <= top_k <= min(E, 32), T*top_k < 2^31;
 *    H and I multiples of 8 (multiples of 128 for MOE_W_INT4_G128,
 *    MOE_W_MXFP8 and MOE_W_MXFP4).
 *  - Weight scales are passed as untyped pointers: bf16 [rows, K/128] for
 *    MOE_W_INT4_G128, E8M0 bytes [rows, K/32] for MOE_W_MXFP8 and
 *    MOE_W_MXFP4, NULL for bf16. Device pointers must be 16-byte aligned
 *    (32-byte for MOE_W_MXFP4 weights; 4-byte for logits/topk_w and the
 *    int32 arrays).
 *  - Pair ids: p = t*K + j for token t and slot j, with K = top_k +
 *    n_shared slots per token. Routed slot order is descending logit; equal
 *    logits go to the lower expert id; shared slots follow.
 *  - Below, "T*top_k" and "E" in array sizes of permute, the GEMMs and
 *    finalize mean T*(top_k + n_shared) and E + n_shared.
 *  - No C++ exception crosses this interface. Entry points are reentrant
 *    given distinct workspaces and outputs.
 *  - The library keeps, per device, the device address of its error flag
 *    (and of moe_permute_noalloc's scratch array), looked up on first use.
 *    These belong to the device's context: do not call the library again
 *    after a cudaDeviceReset in the same process.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,          /* null pointer, bad size, misalignment */
    MOE_ERR_UNSUPPORTED = 2,          /* valid but outside the library's limits */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes below the matching *_workspace_size */
    MOE_ERR_CUDA = 4,                 /* a CUDA runtime/driver call failed */
    MOE_ERR_DEVICE_FLAG = 5           /* reserved: kernels report through the device error
                                         flag, which moe_get_device_error() reads */
} moe_status_t;

typedef enum {
    MOE_W_BF16 = 0,        /* bf16 weights */
    MOE_W_INT4_G128 = 1,   /* W4A16: int4 weights, one bf16 scale per 128 K */
    MOE_W_MXFP8 = 2,       /* MXFP8 (OCP MX v1.0): E4M3 weights, one E8M0 scale per 32 K;
                              the activations are MX-quantised by the layer */
    MOE_W_MXFP4 = 3        /* MXFP4 weights (OCP MX v1.0 E2M1, two per byte, even K in the
                              low nibble, one E8M0 scale per 32 K) with MXFP8 activations */
} moe_weight_fmt_t;

/* Layer shape. T tokens, hidden size H, expert intermediate size I, E routed
 * experts, top_k routed experts per token, fmt a moe_weight_fmt_t, n_shared
 * shared experts (set it to 0 when there are none).
 *
 * Shared experts (GC-MoE abstract: MoE layers with shared experts next to the
 * routed ones): every token also goes through experts E .. E+n_shared-1 of
 * the weight arrays, whose outputs are added with weight 1:
 *   out[t] = sum_{j<top_k} w_j FFN_{e_j}(x_t) + sum_{s<n_shared} FFN_{E+s}(x_t)
 * They are carried as extra slots of each token: the routing arrays are
 * [T, top_k + n_shared], slot top_k + s holds expert E + s with weight 1.0,
 * and permute, the grouped GEMMs and finalize see E + n_shared experts and
 * top_k + n_shared slots. The finalize sum therefore adds the shared
 * experts after the routed slots, in slot order.
 * Limits: top_k + n_shared <= 32 and E + n_shared <= 1024. */
typedef struct {
    int32_t T, H, I, E, top_k, fmt, n_shared;
} moe_shape_t;

typedef uint16_t moe_bf16_t;   /* bit pattern of a bfloat16 value */
typedef void *moe_stream_t;    /* cudaStream_t */

/* Bytes of device workspace moe_forward needs for this shape (0 if the shape
 * is invalid). It holds the intermediates between the steps of InfiniLM PR
 * #500 report §2.2 (routing ids and weights, per-expert counts and offsets,
 * the permutation and its inverse, act [T*k,I] between the gate/up and down
 * grouped GEMMs, y [T*k,H] before the weighted scatter back) and, when many
 * tokens share each expert, the gathered rows [T*k,H] of §2.2 step 2. */
MOE_API size_t moe_workspace_size(const moe_shape_t *shape);

/* Bytes of scratch moe_permute needs (may be 0). */
MOE_API size_t moe_permute_workspace_size(const moe_shape_t *shape);

/* Route. InfiniLM PR #500 report §2.1/§2.4 (top-k softmax routing) with
 * renormalisation over the selected experts.
 *   logits   [T,E] fp32 (NaN ranks as -inf; -0 equals +0)
 *   topk_ids [T,top_k+n_shared] int32 out: expert ids in slot order, then
 *            E .. E+n_shared-1
 *   topk_w   [T,top_k+n_shared] fp32 out: w_j = exp(l_j - l_0) /
 *            sum_i exp(l_i - l_0) over the routed slots (they sum to one;
 *            one warp per token, expf, fp32 sum in slot order), then 1.0 for
 *            each shared slot. */
MOE_API moe_status_t moe_route(const float *logits, const moe_shape_t *shape,
                       int32_t *topk_ids, float *topk_w, moe_stream_t stream);

/* Permute (bucketing). InfiniLM PR #500 report §2.2 step 1 (per-expert counts
 * and a permutation) and step 2 (gather by that permutation), done on the
 * device with no host synchronisation.
 *   topk_ids    [T*top_k] int32 expert ids (0 <= id < E)
 *   counts      [E] out: pairs routed to each expert
 *   offsets     [E+1] out: exclusive prefix sum of counts; offsets[E] = T*top_k
 *   perm        [T*top_k] out: perm[r] = pair id of permuted row r; rows of one
 *               expert are contiguous and in ascending pair id (stable)
 *   inv_perm    [T*top_k] out: inv_perm[perm[r]] = r
 *   hidden      [T,H] bf16, may be NULL (then hidden_perm must be NULL)
 *   hidden_perm [T*top_k,H] bf16 out, may be NULL: hidden_perm[r] = hidden[perm[r]/top_k]
 *   ws, ws_bytes scratch of at least moe_permute_workspace_size() bytes.
 * Deterministic. An id outside [0,E) raises the device error flag; that pair
 * is then dropped (inv_perm = -1) and the sums above no longer hold. */
MOE_API moe_status_t moe_permute(const int32_t *topk_ids, const moe_shape_t *shape,
                         int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                         const moe_bf16_t *hidden, moe_bf16_t *hidden_perm,
                         void *ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped GEMM gate/up with fused SwiGLU. InfiniLM PR #500 report §2.2 step 2
 * (grouped GEMM over all experts in one call, then SwiGLU); FlashInfer PR
 * #7196 analysis §2 (tokens on the MMA N side with a runtime N per tile).
 *   a       perm == NULL: [T*top_k,H] bf16 rows in permuted order (hidden_perm).
 *           perm != NULL: hidden [T,H] bf16; row r of the operand is
 *           a[perm[r] / top_k], gathered inside the GEMM (TMA gather4), so
 *           the permuted copy is never written.
 *   perm    NULL, or [T*top_k] from moe_permute
 *   offsets [E+1] from moe_permute
 *   w_gu    MOE_W_BF16: [E,2I,H] bf16, rows [0,I) gate, rows [I,2I) up.
 *           MOE_W_INT4_G128: [E,2I,H/2] bytes, low nibble = even K index,
 *           two's complement int4; w_gu_scales [E,2I,H/128] bf16.
 *           w = bf16(q * scale) is formed on chip (in tensor memory, the
 *           MMA's A operand) before the MMA; it never reaches HBM.
 *   act     [T*top_k,I] bf16 out: act = bf16(silu(g) * u), g/u fp32 accumulated.
 * Experts with no rows cost no tiles. */
MOE_API moe_status_t moe_grouped_gemm_swiglu(const moe_bf16_t *a, const int32_t *perm, const int32_t *offsets,
                                     const void *w_gu, const void *w_gu_scales,
                                     const moe_shape_t *shape, moe_bf16_t *act, moe_stream_t stream);

/* Grouped GEMM down. InfiniLM PR #500 report §2.2 step 2 (third grouped GEMM).
 *   act     [T*top_k,I] bf16, offsets [E+1]
 *   w_d     MOE_W_BF16: [E,H,I] bf16. MOE_W_INT4_G128: [E,H,I/2] bytes with
 *           w_d_scales [E,H,I/128] bf16; w = bf16(q * scale) is formed on
 *           chip (in tensor memory, or, with at most 24 rows per expert on
 *           average, in the registers that feed warp-level MMAs) and never
 *           reaches HBM.
 *   y       [T*top_k,H] bf16 out: unscaled down projection, permuted row order. */
MOE_API moe_status_t moe_grouped_gemm_down(const moe_bf16_t *act, const int32_t *offsets,
                                   const void *w_d, const void *w_d_scales,
                                   const moe_shape_t *shape, moe_bf16_t *y, moe_stream_t stream);

/* Finalize / unpermute. FlashInfer PR #7196 analysis §1 (moe_finalize):
 *   out[t,h] = bf16_rne(acc), acc = v_0 * w_0 (fp32 multiply, round to
 *   nearest), then acc = fma(v_j, w_j, acc) for j = 1..top_k-1 (round to
 *   nearest, no flush-to-zero), v_j = y[inv_perm[t*top_k+j], h],
 *   w_j = topk_w[t*top_k+j]. Signed zeros and subnormals are kept.
 *   A row index outside [0, T*top_k) reads as 0 and raises device error 3
 *   (moe_get_device_error). Bit-exact and deterministic. */
MOE_API moe_status_t moe_finalize(const moe_bf16_t *y, const float *topk_w, const int32_t *inv_perm,
                          const moe_shape_t *shape, moe_bf16_t *out, moe_stream_t stream);

/* Number of kernels moe_forward enqueues for this shape (0 when T = 0, -1
 * when the shape is invalid). Host-side only; launches nothing. */
MOE_API int32_t moe_forward_kernel_count(const moe_shape_t *shape);

/* 1 when moe_forward runs this shape as moe_forward_fused (one persistent
 * kernel after a counter reset), 0 when it runs the step kernels, -1 for an
 * invalid shape. Host-side only. */
MOE_API int32_t moe_forward_is_fused(const moe_shape_t *shape);

/* 1 when moe_forward's gate/up GEMM reads the token rows through perm itself
 * (no gathered copy is written), 0 when it gathers first, -1 for an invalid
 * shape. The same choice for moe_grouped_gemm_swiglu with a non-NULL perm
 * runs the kernel moe_forward runs. Host-side only. */
MOE_API int32_t moe_forward_gathers_in_gemm(const moe_shape_t *shape);

/* The whole layer, in the order of InfiniLM PR #500 report §2.2 (bucket the
 * routing indices, gather, grouped GEMMs gate/up and down with SwiGLU between
 * them, scale by the routing weights and scatter back) with the routing of
 * §2.1/§2.4 and the finalize arithmetic of FlashInfer PR #7196 analysis §1:
 * route, permute (with the gather when many tokens share each expert;
 * otherwise the gate/up GEMM gathers through perm itself), gate/up + SwiGLU,
 * down, finalize, enqueued on one stream with no host synchronisation. The
 * result equals the step entry points called in that order. A decode batch
 * with bf16 weights (the shapes moe_forward_fused takes, moe_forward_is_fused
 * says which) runs as moe_forward_fused: the same result in one persistent
 * kernel.
 *   hidden [T,H] bf16, logits [T,E] fp32, weights as above, out [T,H] bf16.
 *   ws: at least moe_workspace_size(shape) bytes, 256-byte aligned; the
 *   call overwrites it, so calls that overlap on the GPU need distinct
 *   workspaces. */
MOE_API moe_status_t moe_forward(const moe_bf16_t *hidden, const float *logits,
                         const void *w_gu, const void *w_gu_scales,
                         const void *w_d, const void *w_d_scales,
                         const moe_shape_t *shape, moe_bf16_t *out,
                         void *ws, size_t ws_bytes, moe_stream_t stream);

/* The whole layer for a decode batch in ONE persistent kernel: routing,
 * bucketing, gate/up + SwiGLU, down and finalize, with no kernel boundary
 * between them (the GC-MoE abstract fuses the layer's steps into one graph;
 * the steps and their arithmetic are those of moe_forward, which it equals
 * bit for bit on these shapes). Every CTA routes and buckets the batch in
 * shared memory and takes tiles from a counter in the workspace; a down
 * tile loads act once its expert's gate/up tiles have finished and finalize
 * starts once every down tile has (counters in the workspace, bounded
 * waits). A one-warp kernel zeroes the counters first: two kernels in all,
 * both with programmatic dependent launch.
 *   bf16 weights, 1 <= T <= 64, top_k + n_shared <= 16, E + n_shared <= 256;
 *   other shapes return MOE_ERR_UNSUPPORTED before anything is enqueued.
 *   ws: at least moe_workspace_size(shape) bytes, 256-byte aligned; it also
 *   holds the routing and the permutation of the call (as moe_forward's). */
MOE_API moe_status_t moe_forward_fused(const moe_bf16_t *hidden, const float *logits, const void *w_gu,
                                       const void *w_d, const moe_shape_t *shape, moe_bf16_t *out, void *ws,
                                       size_t ws_bytes, moe_stream_t stream);

/* moe_forward with hidden, logits and out in HOST memory (page-locked memory
 * gives asynchronous copies). Copies the inputs into the workspace, runs the
 * layer and copies out back, then waits: when it returns OK, out_host holds
 * the result. Weights stay device-resident. Up to 2047 tokens everything runs
 * on `stream`. Larger batches are cut into 2 to 4 chunks of at least 1024
 * tokens. The inputs of one chunk are copied in, and the output of the one
 * before is copied out, on two streams the library creates once per device,
 * while `stream` computes the current chunk. Each token's result depends only
 * on its own row, so the output is the same bits. Calls on one device take
 * turns on those streams, and a cudaDeviceReset invalidates them.
 *   ws: at least moe_forward_host_workspace_size(shape) bytes. */
MOE_API size_t moe_forward_host_workspace_size(const moe_shape_t *shape);
MOE_API moe_status_t moe_forward_host(const moe_bf16_t *hidden_host, const float *logits_host,
                              const void *w_gu, const void *w_gu_scales,
                              const void *w_d, const void *w_d_scales,
                              const moe_shape_t *shape, moe_bf16_t *out_host,
                              void *ws, size_t ws_bytes, moe_stream_t stream);

/* MXFP8 (OCP Microscaling Formats (MX) v1.0; the GC-MoE abstract runs its
 * expert GEMMs in FP8 / FP4). The block-scaled tensor-core MMA
 * (tcgen05.mma kind::mxf8f6f4) takes both operands in MX form, so with
 * MOE_W_MXFP8 weights the layer MX-quantises its activations: hidden before
 * gate/up, and act (after its bf16 rounding) before down. moe_forward does
 * all of it; these are the steps on their own.
 *
 * Quantisation of x [rows, K] bf16 (K % 32 == 0) into q [rows, K] E4M3 and
 * scales [rows, K/32] E8M0: per block of 32 consecutive elements, e =
 * floor(log2 max|x|) - 8 clamped to [-127, 127] (-127 for an all-zero
 * block; the scale byte is e + 127), then q = E4M3(x / 2^e), rounded to
 * nearest even and saturated to +-448. Bit-exact. */
MOE_API moe_status_t moe_mx_quantize(const moe_bf16_t *x, int32_t rows, int32_t K, uint8_t *q, uint8_t *scales,
                                     moe_stream_t stream);

/* Gate/up + SwiGLU with MXFP8 or MXFP4 weights (shape->fmt = MOE_W_MXFP8
 * or MOE_W_MXFP4; the token operand is MXFP8 either way):
 *   a_q, a_scales  perm == NULL: permuted rows [T*top_k, H] / [T*top_k, H/32];
 *                  perm != NULL: hidden's quantisation [T, H] / [T, H/32], rows
 *                  read through perm (TMA gather4)
 *   w_gu MOE_W_MXFP8: [E,2I,H] E4M3; MOE_W_MXFP4: [E,2I,H/2] packed E2M1;
 *        w_gu_scales [E,2I,H/32] E8M0
 *   act_q [T*top_k, I] E4M3 and act_scales [T*top_k, I/32] out: the MX
 *   quantisation of act = bf16(silu(g) * u), fp32 accumulation. */
MOE_API moe_status_t moe_grouped_gemm_swiglu_mx(const uint8_t *a_q, const uint8_t *a_scales, const int32_t *perm,
                                                const int32_t *offsets, const void *w_gu, const void *w_gu_scales,
                                                const moe_shape_t *shape, uint8_t *act_q, uint8_t *act_scales,
                                                moe_stream_t stream);

/* Down with MXFP8 or MXFP4 weights: act_q [T*top_k, I] E4M3 + act_scales
 * [T*top_k, I/32], w_d [E,H,I] E4M3 (MXFP4: [E,H,I/2] packed E2M1) +
 * w_d_scales [E,H,I/32] -> y [T*top_k, H] bf16. */
MOE_API moe_status_t moe_grouped_gemm_down_mx(const uint8_t *act_q, const uint8_t *act_scales,
                                              const int32_t *offsets, const void *w_d, const void *w_d_scales,
                                              const moe_shape_t *shape, moe_bf16_t *y, moe_stream_t stream);

/* W4A16 weight decoding on its own (the step the int4 GEMMs run on chip
 * before their MMAs). FlashInfer PR #7196 analysis §2-§3.
 *   q [rows, K/2] bytes, scales [rows, K/128] bf16 -> out [rows, K] bf16,
 *   out = bf16_rne(q * scale). K a multiple of 128. */
MOE_API moe_status_t moe_dequant_int4(const uint8_t *q, const moe_bf16_t *scales, int32_t rows, int32_t K,
                              moe_bf16_t *out, moe_stream_t stream);

/* Device error flag of the current device: waits for all work on the device,
 * stores the flag in *code (0 = none; 1 = bad expert id; 2 = a pipeline wait
 * timed out; 3 = a finalize row index out of range; 4 = a permutation entry
 * or an expert offset out of range, caught only by the range-checking build
 * libmoe_b200_debug.so, compiled from the same sources with
 * -DMOE_DEBUG_BOUNDS, which then uses an in-range value instead) and clears
 * it. The first error raised since the last read is the one kept. */
MOE_API moe_status_t moe_get_device_error(int32_t *code);

/* Self-test of the bounded waits behind device error code 2 (no counterpart
 * on the pages). Enqueues one CTA that waits on a pipeline barrier that
 * nothing ever arrives on; after limit_ns nanoseconds of %globaltimer the
 * wait gives up, sets the device error flag to 2 and the kernel returns.
 * Nothing faults or traps and the context stays usable: a following
 * moe_get_device_error() reads 2 and clears it.
 *   limit_ns  1 .. 1e9 (one second at most), else MOE_ERR_INVALID_ARG
 *             and nothing is enqueued. */
MOE_API moe_status_t moe_selftest_bounded_wait(int64_t limit_ns, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory: the same
 * outputs, bit for bit, with the scratch taken from a fixed 256 KiB array
 * built into the library instead of a caller workspace. It is meant for code
 * that runs inside a host framework which owns every device allocation and
 * passes no workspace, and for hot loops that must not call cudaMalloc,
 * because that call can synchronise the device. The pages have no
 * counterpart to this entry point.
 *   Arguments as moe_permute, without ws/ws_bytes. It allocates nothing and
 *   calls no allocating routine.
 *   Limit: the per-chunk histogram, ceil(T*top_k / 2048) * E int32 entries,
 *   must fit 65536 entries. For example, E = 128 allows up to 1,048,576
 *   pairs. Larger calls return MOE_ERR_UNSUPPORTED before anything is
 *   enqueued. Calls with T*top_k <= 8192 use no scratch at all.
 *   The array exists once per GPU that loads the library and is held until
 *   the process exits. Its device address is looked up on the first call
 *   made with a given device current, so make that first call before any
 *   stream capture.
 *   Every call on a device shares the one array. Calls whose work overlaps
 *   on the GPU (different streams, no ordering between them) race on it, so
 *   order such calls. Each call overwrites every entry it reads, so the
 *   previous call's contents need no clearing. */
MOE_API moe_status_t moe_permute_noalloc(const int32_t *topk_ids, const moe_shape_t *shape,
                                         int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                         const moe_bf16_t *hidden, moe_bf16_t *hidden_perm,
                                         moe_stream_t stream);

/* ---- Expert parallelism ------------------------------------------------------
 * The experts split over `world` ranks (rank d owns experts d*E/world ..
 * (d+1)*E/world - 1, and their weights), each rank holding its own tokens
 * (GC-MoE abstract: experts partitioned over GPUs, tokens dispatched to their
 * experts' GPU and the outputs combined back). The steps write straight into
 * other ranks' buffers through the pointers of moe_ep_peers_t: buffers of the
 * same GPU, or of peer GPUs with peer access enabled (the stores then cross
 * NVLink). No kernel waits for another rank; between the phases the caller
 * puts a barrier over all ranks (marked | below). On each rank r, with
 * shape = {T_r tokens, H, I, E all routed experts, top_k, fmt, n_shared 0}:
 *   moe_route, moe_permute (counts, offsets, perm, inv_perm over all E)
 *   moe_ep_count                          |
 *   moe_ep_dispatch                       |
 *   moe_ep_local_offsets, then moe_grouped_gemm_swiglu and _down on
 *     recv_rows[r] (perm NULL, the local offsets, the E/world local experts'
 *     weights, a shape with E = E/world and T*top_k >= the rows received)
 *   moe_ep_combine                        |
 *   moe_finalize(y_ret[r], topk_w, identity inv_perm) -> out.
 * Every pair's arithmetic is moe_forward's on rank r's own tokens; the
 * result equals it bit for bit.
 * Receive buffer of rank d: rows grouped by d's local expert, then by source
 * rank, then in the source's permutation order; recv_src holds each row's
 * origin as (source rank << 24) | pair id. */
#define MOE_EP_MAX_RANKS 8
typedef struct {
    int32_t world;                                /* ranks, 1 .. MOE_EP_MAX_RANKS */
    int32_t rank;                                 /* this rank */
    int32_t capacity;                             /* rows of every receive buffer */
    int32_t *counts[MOE_EP_MAX_RANKS];            /* rank d: [world, E/world] int32: row s = pairs of
                                                     source s per local expert */
    moe_bf16_t *recv_rows[MOE_EP_MAX_RANKS];      /* rank d: [capacity, H] bf16, 16-byte aligned */
    int32_t *recv_src[MOE_EP_MAX_RANKS];          /* rank d: [capacity] origins */
    moe_bf16_t *y_ret[MOE_EP_MAX_RANKS];          /* rank r: [T_r*top_k, H] bf16: the down output of
                                                     each of r's pairs, at its pair id */
    int32_t pairs[MOE_EP_MAX_RANKS];              /* rank r: T_r*top_k, the rows of y_ret[r] */
} moe_ep_peers_t;

/* This rank's pairs per expert (from its offsets [E+1]) into row `rank` of
 * every owner's counts; zeros when this rank has no tokens (T = 0: offsets
 * are not read and may be NULL). Unlike the other entry points it runs for
 * T = 0, since the other ranks need this rank's row. */
MOE_API moe_status_t moe_ep_count(const int32_t *offsets, const moe_shape_t *shape, const moe_ep_peers_t *peers,
                                  moe_stream_t stream);
/* After every rank's count: this rank's permuted rows (hidden [T,H] through
 * perm [T*top_k], offsets [E+1]) into their owners' receive buffers. A row
 * past `capacity` is not written and raises device error 4. */
MOE_API moe_status_t moe_ep_dispatch(const moe_bf16_t *hidden, const int32_t *perm, const int32_t *offsets,
                                     const moe_shape_t *shape, const moe_ep_peers_t *peers, moe_stream_t stream);
/* After every rank's dispatch: offsets_local [E/world + 1] of this rank's
 * receive buffer over its local experts (offsets_local[E/world] = rows
 * received). */
MOE_API moe_status_t moe_ep_local_offsets(const moe_shape_t *shape, const moe_ep_peers_t *peers,
                                          int32_t *offsets_local, moe_stream_t stream);
/* After the local GEMMs: y_local [capacity, H] (the down output of this
 * rank's received rows) back to each row's source, into y_ret[source] at the
 * row's pair id (a pair id at or past pairs[source] raises device error 4 and
 * is skipped). */
MOE_API moe_status_t moe_ep_combine(const moe_bf16_t *y_local, const int32_t *offsets_local,
                                    const moe_shape_t *shape, const moe_ep_peers_t *peers, moe_stream_t stream);

/* Static description of a status code. */
MOE_API const char *moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
