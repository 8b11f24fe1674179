// capi.cu -- the extern "C" entry points of libmoe_b200 (declared and
// documented in include/moe.h): argument validation, workspace layout and the
// launch sequence of the whole layer. Compute lives in the kernel files.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <memory>
#include <mutex>

#include "launch.h"
#include "moe.h"

// Device error flag word (0 = none), one per device that loads the library.
static __device__ int g_moe_error_flag;

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_moe_error_flag on the current device, looked up on the
// first call made with that device current. Concurrent first calls may both
// look it up; they store the same address. The cached address belongs to the
// device's context, so the library must not be used across a cudaDeviceReset.
int *error_flag_ptr() {
    static std::atomic<int *> ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int *p = ptrs[dev].load(std::memory_order_acquire);
    if (!p) {
        void *q = nullptr;
        if (cudaGetSymbolAddress(&q, g_moe_error_flag) != cudaSuccess) return nullptr;
        p = static_cast<int *>(q);
        ptrs[dev].store(p, std::memory_order_release);
    }
    return p;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Slots per token (routed, then shared) and experts in the weight arrays.
inline int slots(const moe_shape_t *s) { return s->top_k + s->n_shared; }
inline int experts(const moe_shape_t *s) { return s->E + s->n_shared; }
// Block-scaled formats: MX weights, MXFP8 activations.
inline bool is_mx(int fmt) { return fmt == MOE_W_MXFP8 || fmt == MOE_W_MXFP4; }

moe_status_t check_shape(const moe_shape_t *s) {
    if (!s) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->H <= 0 || s->I <= 0 || s->E < 1 || s->top_k < 1 || s->top_k > s->E || s->n_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (s->fmt != MOE_W_BF16 && s->fmt != MOE_W_INT4_G128 && s->fmt != MOE_W_MXFP8 && s->fmt != MOE_W_MXFP4)
        return MOE_ERR_INVALID_ARG;
    if (static_cast<long long>(s->E) + s->n_shared > 1024 || static_cast<long long>(s->top_k) + s->n_shared > 32)
        return MOE_ERR_UNSUPPORTED;
    if (s->H % 8 || s->I % 8) return MOE_ERR_UNSUPPORTED;
    if (s->fmt != MOE_W_BF16 && (s->H % 128 || s->I % 128)) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(s->T) * slots(s) >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(experts(s)) * 2 * s->I >= (1LL << 31) ||
        static_cast<long long>(experts(s)) * s->H >= (1LL << 31))
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte offsets of moe_forward's intermediates inside the workspace.
struct Layout {
    size_t ids, w, counts, offsets, perm, inv, scratch, hperm, act, y;
    size_t hq, hs, aq, as;                 // MX formats: hidden and act, E4M3 codes and E8M0 scales
    size_t done;                           // moe_forward_fused: per-expert and finish counters
    size_t hidden_in, logits_in, out_st;   // staging for moe_forward_host
    size_t total;
};

Layout layout(const moe_shape_t *s, bool host) {
    const size_t P = static_cast<size_t>(s->T) * slots(s);
    const int E = experts(s);
    Layout L;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align256(o + bytes);
        return at;
    };
    L.ids = take(P * 4);
    L.w = take(P * 4);
    L.counts = take(static_cast<size_t>(E) * 4);
    L.offsets = take(static_cast<size_t>(E + 1) * 4);
    L.perm = take(P * 4);
    L.inv = take(P * 4);
    L.scratch = take(moe::permute_scratch_bytes(static_cast<long long>(P), E));
    L.hperm = moe::gemm_gathers_in_kernel(static_cast<int>(P), E, s->fmt) ? o : take(P * s->H * 2);
    const bool mx = is_mx(s->fmt);
    L.act = mx ? o : take(P * s->I * 2);
    L.y = take(P * s->H * 2);
    L.hq = L.hs = L.aq = L.as = o;
    if (mx) {
        L.hq = take(static_cast<size_t>(s->T) * s->H);
        L.hs = take(static_cast<size_t>(s->T) * s->H / 32);
        L.aq = take(P * s->I);
        L.as = take(P * s->I / 32);
    }
    L.done = take(moe::fused_counter_words(s->E, s->n_shared) * 4);
    L.hidden_in = L.logits_in = L.out_st = 0;
    if (host) {
        L.hidden_in = take(static_cast<size_t>(s->T) * s->H * 2);
        L.logits_in = take(static_cast<size_t>(s->T) * s->E * 4);
        L.out_st = take(static_cast<size_t>(s->T) * s->H * 2);
    }
    L.total = o;
    return L;
}

moe::GemmArgs gemm_args(const moe_shape_t *s, const void *a, const int32_t *perm, const int32_t *offsets,
                        const void *w, const void *scales, bool swiglu, moe_bf16_t *out) {
    moe::GemmArgs g;
    g.a = a;
    g.perm = perm;
    g.T = s->T;
    g.top_k = slots(s);
    g.offsets = offsets;
    g.w = w;
    g.w_scales = s->fmt == MOE_W_INT4_G128 ? static_cast<const uint16_t *>(scales) : nullptr;
    g.P = s->T * slots(s);
    g.E = experts(s);
    g.K = swiglu ? s->H : s->I;
    g.m_out = swiglu ? s->I : s->H;
    g.w_rows = swiglu ? 2 * s->I : s->H;
    g.fmt = s->fmt;
    g.swiglu = swiglu;
    g.out = out;
    g.err = error_flag_ptr();
    return g;
}

moe_status_t check_weights(const moe_shape_t *s, const void *w, const void *scales) {
    // MXFP4 weights are read by TMA as packed 4-bit elements: 32-byte aligned
    if (!w || !aligned(w, s->fmt == MOE_W_MXFP4 ? 32 : 16)) return MOE_ERR_INVALID_ARG;
    if (s->fmt != MOE_W_BF16) {
        if (!scales || !aligned(scales, 4)) return MOE_ERR_INVALID_ARG;
    } else if (scales) {
        return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

// The MXFP8 GEMM arguments: token rows a_q (E4M3) with scales a_sf, weight
// scales w_sf, gate/up output act_q / act_sf (E4M3 / E8M0) or down output y.
moe::MxGemmArgs mx_args(const moe_shape_t *s, const uint8_t *a_q, const uint8_t *a_sf, const int32_t *perm,
                        const int32_t *offsets, const void *w, const void *w_sf, bool swiglu, uint8_t *act_q,
                        uint8_t *act_sf, moe_bf16_t *y) {
    moe::MxGemmArgs m;
    m.base = gemm_args(s, a_q, perm, offsets, w, nullptr, swiglu, y);
    m.w_sf = static_cast<const uint8_t *>(w_sf);
    m.x_sf = a_sf;
    m.out_q = act_q;
    m.out_sf = act_sf;
    return m;
}

moe_status_t forward_device(const moe_bf16_t *hidden, const float *logits, const void *w_gu,
                            const void *w_gu_scales, const void *w_d, const void *w_d_scales,
                            const moe_shape_t *s, moe_bf16_t *out, uint8_t *ws, const Layout &L,
                            cudaStream_t st) {
    // routing: top_k of the E routed experts, then the shared slots; every
    // later step sees K = top_k + n_shared slots over E + n_shared experts
    const int T = s->T, kr = s->top_k, Er = s->E, S = s->n_shared, H = s->H;
    const int k = slots(s), E = experts(s);
    const int P = T * k;
    auto *ids = reinterpret_cast<int32_t *>(ws + L.ids);
    auto *w = reinterpret_cast<float *>(ws + L.w);
    auto *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    auto *offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    auto *perm = reinterpret_cast<int32_t *>(ws + L.perm);
    auto *inv = reinterpret_cast<int32_t *>(ws + L.inv);
    auto *act = reinterpret_cast<uint16_t *>(ws + L.act);
    auto *y = reinterpret_cast<uint16_t *>(ws + L.y);
    // a decode batch with bf16 weights: the whole layer in one persistent kernel
    if (moe::fused_decode_supported(T, H, s->I, Er, kr, S, s->fmt))
        return cuda_status(moe::launch_fused_decode(logits, hidden, w_gu, w_d, T, H, s->I, Er, kr, S, ids, w, counts,
                                                    offsets, perm, inv, act, y, out,
                                                    reinterpret_cast<unsigned int *>(ws + L.done), error_flag_ptr(),
                                                    st));
    cudaError_t e;
    if (moe::route_permute_fusable(T, E, k)) {
        e = moe::launch_route_permute(logits, T, Er, kr, S, ids, w, counts, offsets, perm, inv, error_flag_ptr(), st);
        if (e != cudaSuccess) return cuda_status(e);
    } else {
        if ((e = moe::launch_route(logits, T, Er, kr, S, ids, w, st)) != cudaSuccess) return cuda_status(e);
        if ((e = moe::launch_permute(ids, P, E, counts, offsets, perm, inv, ws + L.scratch, error_flag_ptr(), st)) !=
            cudaSuccess)
            return cuda_status(e);
    }
    if (is_mx(s->fmt)) {
        // MX weights: hidden quantised once per token; gate/up gathers its rows through
        // perm and writes act quantised; down reads act's codes and scales
        auto *hq = ws + L.hq, *hs = ws + L.hs, *aq = ws + L.aq, *as = ws + L.as;
        if ((e = moe::launch_mx_quantize(hidden, T, H, hq, hs, st)) != cudaSuccess) return cuda_status(e);
        e = moe::launch_grouped_gemm_mxfp8(mx_args(s, hq, hs, perm, offsets, w_gu, w_gu_scales, true, aq, as, nullptr),
                                           st);
        if (e != cudaSuccess) return cuda_status(e);
        e = moe::launch_grouped_gemm_mxfp8(mx_args(s, aq, as, nullptr, offsets, w_d, w_d_scales, false, nullptr,
                                                   nullptr, y), st);
        if (e != cudaSuccess) return cuda_status(e);
        return cuda_status(moe::launch_finalize(y, w, inv, T, H, k, out, error_flag_ptr(), st));
    }
    // Few rows per expert: the gate/up GEMM gathers the token rows itself (TMA
    // gather4 through perm). Many rows per expert: one gather kernel writes the
    // permuted rows and the GEMM reads them as whole 128-row tiles, which keeps
    // its TMA unit from turning into the bottleneck.
    if (moe::gemm_gathers_in_kernel(P, E, s->fmt)) {
        moe::GemmArgs gu = gemm_args(s, hidden, perm, offsets, w_gu, w_gu_scales, true, act);
        gu.hints = moe::kGemmHintPrefetchGuess;     // routing runs on few SMs: warm L2 meanwhile
        e = moe::launch_grouped_gemm(gu, st);
    } else {
        auto *hperm = reinterpret_cast<uint16_t *>(ws + L.hperm);
        if ((e = moe::launch_gather(hidden, perm, P, H, k, hperm, error_flag_ptr(), st)) != cudaSuccess) return cuda_status(e);
        e = moe::launch_grouped_gemm(gemm_args(s, hperm, nullptr, offsets, w_gu, w_gu_scales, true, act), st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    // offsets were complete before the gate/up GEMM started, so the down GEMM
    // may start loading weights while gate/up finishes
    moe::GemmArgs dn = gemm_args(s, act, nullptr, offsets, w_d, w_d_scales, false, y);
    dn.hints = moe::kGemmHintOffsetsReady;
    if ((e = moe::launch_grouped_gemm(dn, st)) != cudaSuccess) return cuda_status(e);
    return cuda_status(moe::launch_finalize(y, w, inv, T, H, k, out, error_flag_ptr(), st));
}

// ---- moe_forward_host for large batches: chunks in a copy/compute pipeline ----
// Each token's output depends only on its own row, so the batch can be cut
// into chunks of tokens without changing a bit. Chunk c's inputs are copied
// in on one library stream while chunk c-1 computes on the caller's stream,
// and chunk c-1's output is copied out on another while chunk c computes.
constexpr int kHostChunkTokens = 1024;   // smallest chunk
constexpr int kHostMaxChunks = 4;

int host_chunks(const moe_shape_t *s) {
    const int c = s->T / kHostChunkTokens;
    return c < 2 ? 1 : (c < kHostMaxChunks ? c : kHostMaxChunks);
}

// The two copy streams and the events of one device, created on first use
// and kept for the process; a call holds `m` from its first copy to its end.
struct HostPipe {
    std::mutex m;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, in_done[kHostMaxChunks] = {}, comp_done[kHostMaxChunks] = {};
    bool ready = false;
};

HostPipe *host_pipe(int dev) {
    static std::mutex mu;
    static std::map<int, std::unique_ptr<HostPipe>> pipes;
    std::lock_guard<std::mutex> lock(mu);
    auto &p = pipes[dev];
    if (!p) p.reset(new HostPipe());
    return p.get();
}

moe_status_t forward_host_chunked(const moe_bf16_t *hidden_host, const float *logits_host, const void *w_gu,
                                  const void *w_gu_scales, const void *w_d, const void *w_d_scales,
                                  const moe_shape_t *shape, moe_bf16_t *out_host, uint8_t *base, const Layout &L,
                                  cudaStream_t s) {
    const int C = host_chunks(shape);
    const int Tc = (shape->T + C - 1) / C;
    moe_shape_t cs = *shape;
    cs.T = Tc;
    const Layout Lc = layout(&cs, false);            // a chunk's intermediates, inside the full layout's
    if (Lc.total > L.hidden_in) return MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    HostPipe *hp = host_pipe(dev);
    std::lock_guard<std::mutex> lock(hp->m);
    if (!hp->ready) {
        bool ok = cudaStreamCreateWithFlags(&hp->in, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&hp->out, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&hp->start, cudaEventDisableTiming) == cudaSuccess;
        for (int c = 0; ok && c < kHostMaxChunks; ++c)
            ok = cudaEventCreateWithFlags(&hp->in_done[c], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&hp->comp_done[c], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return MOE_ERR_CUDA;
        hp->ready = true;
    }
    const size_t H = shape->H, E = shape->E;
    // the copies start after the work already on the caller's stream
    if (cudaEventRecord(hp->start, s) != cudaSuccess || cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    for (int c = 0; c < C; ++c) {
        const size_t t0 = static_cast<size_t>(c) * Tc;
        const int tc = static_cast<int>(std::min<size_t>(Tc, shape->T - t0));
        if (cudaMemcpyAsync(base + L.hidden_in + t0 * H * 2, hidden_host + t0 * H, tc * H * 2,
                            cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
            cudaMemcpyAsync(base + L.logits_in + t0 * E * 4, logits_host + t0 * E, tc * E * 4,
                            cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
            cudaEventRecord(hp->in_done[c], hp->in) != cudaSuccess || cudaStreamWaitEvent(s, hp->in_done[c], 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        cs.T = tc;
        const moe_status_t st = forward_device(
            reinterpret_cast<const moe_bf16_t *>(base + L.hidden_in) + t0 * H,
            reinterpret_cast<const float *>(base + L.logits_in) + t0 * E, w_gu, w_gu_scales, w_d, w_d_scales, &cs,
            reinterpret_cast<moe_bf16_t *>(base + L.out_st) + t0 * H, base, layout(&cs, false), s);
        if (st != MOE_OK) return st;
        if (cudaEventRecord(hp->comp_done[c], s) != cudaSuccess ||
            cudaStreamWaitEvent(hp->out, hp->comp_done[c], 0) != cudaSuccess ||
            cudaMemcpyAsync(out_host + t0 * H, base + L.out_st + t0 * H * 2, tc * H * 2, cudaMemcpyDeviceToHost,
                            hp->out) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // the caller's stream continues after the last copy out; the call returns
    // when everything is done
    if (cudaEventRecord(hp->start, hp->out) != cudaSuccess || cudaStreamWaitEvent(s, hp->start, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(s));
}

}  // namespace

namespace moe {
moe_status_t validate_shape(const moe_shape_t *shape) { return check_shape(shape); }
int shape_slots(const moe_shape_t *shape) { return slots(shape); }
int shape_experts(const moe_shape_t *shape) { return experts(shape); }
int *device_error_flag() { return error_flag_ptr(); }
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return 0;
    return layout(shape, false).total;
}

size_t moe_forward_host_workspace_size(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return 0;
    return layout(shape, true).total;
}

size_t moe_permute_workspace_size(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return 0;
    return moe::permute_scratch_bytes(static_cast<long long>(shape->T) * slots(shape), experts(shape));
}

moe_status_t moe_route(const float *logits, const moe_shape_t *shape, int32_t *topk_ids, float *topk_w,
                       moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_route");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w || !aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_route(logits, shape->T, shape->E, shape->top_k, shape->n_shared, topk_ids,
                                         topk_w, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute(const int32_t *topk_ids, const moe_shape_t *shape, int32_t *counts, int32_t *offsets,
                         int32_t *perm, int32_t *inv_perm, const moe_bf16_t *hidden, moe_bf16_t *hidden_perm,
                         void *ws, size_t ws_bytes, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_permute");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    const long long P = static_cast<long long>(shape->T) * slots(shape);
    const int E = experts(shape);
    if (!counts || !offsets || !aligned(counts, 4) || !aligned(offsets, 4)) return MOE_ERR_INVALID_ARG;
    if (P > 0 && (!topk_ids || !perm || !inv_perm || !aligned(topk_ids, 4) || !aligned(perm, 4) ||
                  !aligned(inv_perm, 4)))
        return MOE_ERR_INVALID_ARG;
    if ((hidden == nullptr) != (hidden_perm == nullptr)) return MOE_ERR_INVALID_ARG;
    if (hidden && (!aligned(hidden, 16) || !aligned(hidden_perm, 16))) return MOE_ERR_INVALID_ARG;
    const size_t need = moe::permute_scratch_bytes(P, E);
    if (need > 0 && (!ws || ws_bytes < need)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (ws && !aligned(ws, 16)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = moe::launch_permute(topk_ids, static_cast<int>(P), E, counts, offsets, perm, inv_perm, ws,
                                        error_flag_ptr(), s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (hidden)
        e = moe::launch_gather(hidden, perm, static_cast<int>(P), shape->H, slots(shape), hidden_perm,
                               error_flag_ptr(), s);
    return cuda_status(e);
}

moe_status_t moe_grouped_gemm_swiglu(const moe_bf16_t *a, const int32_t *perm, const int32_t *offsets,
                                     const void *w_gu, const void *w_gu_scales, const moe_shape_t *shape,
                                     moe_bf16_t *act, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_grouped_gemm_swiglu");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (is_mx(shape->fmt)) return MOE_ERR_UNSUPPORTED;             // moe_grouped_gemm_swiglu_mx
    if (shape->T == 0) return MOE_OK;
    if (!a || !offsets || !act || !aligned(a, 16) || !aligned(act, 16) || !aligned(offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if (perm && !aligned(perm, 4)) return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_gu, w_gu_scales)) != MOE_OK) return st;
    return cuda_status(moe::launch_grouped_gemm(gemm_args(shape, a, perm, offsets, w_gu, w_gu_scales, true, act),
                                                static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_down(const moe_bf16_t *act, const int32_t *offsets, const void *w_d,
                                   const void *w_d_scales, const moe_shape_t *shape, moe_bf16_t *y,
                                   moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_grouped_gemm_down");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (is_mx(shape->fmt)) return MOE_ERR_UNSUPPORTED;             // moe_grouped_gemm_down_mx
    if (shape->T == 0) return MOE_OK;
    if (!act || !offsets || !y || !aligned(act, 16) || !aligned(y, 16) || !aligned(offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_d, w_d_scales)) != MOE_OK) return st;
    return cuda_status(moe::launch_grouped_gemm(gemm_args(shape, act, nullptr, offsets, w_d, w_d_scales, false, y),
                                                static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_finalize(const moe_bf16_t *y, const float *topk_w, const int32_t *inv_perm,
                          const moe_shape_t *shape, moe_bf16_t *out, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_finalize");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!y || !topk_w || !inv_perm || !out || !aligned(y, 16) || !aligned(out, 16) || !aligned(topk_w, 4) ||
        !aligned(inv_perm, 4))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_finalize(y, topk_w, inv_perm, shape->T, shape->H, slots(shape), out,
                                            error_flag_ptr(), static_cast<cudaStream_t>(stream)));
}

int32_t moe_forward_kernel_count(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return -1;
    if (shape->T == 0) return 0;
    const int T = shape->T, k = slots(shape), E = experts(shape);
    const long long P = static_cast<long long>(T) * k;
    if (moe_forward_is_fused(shape) == 1) return 2;                  // counter reset, the persistent kernel
    int32_t n = 0;
    if (moe::route_permute_fusable(T, E, k))
        n += 1;                                                       // route + permute in one CTA
    else
        n += 1 + moe::permute_kernel_count(P, E);                     // route; permute in 1, 2 or 3 kernels
    if (!moe::gemm_gathers_in_kernel(static_cast<int>(P), E, shape->fmt)) n += 1;   // gather
    if (is_mx(shape->fmt)) n += 1;                                    // MX quantisation of hidden
    return n + 3;                                                     // gate/up, down, finalize
}

int32_t moe_forward_is_fused(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return -1;
    return moe::fused_decode_supported(shape->T, shape->H, shape->I, shape->E, shape->top_k, shape->n_shared,
                                       shape->fmt)
               ? 1
               : 0;
}

int32_t moe_forward_gathers_in_gemm(const moe_shape_t *shape) {
    if (check_shape(shape) != MOE_OK) return -1;
    return moe::gemm_gathers_in_kernel(shape->T * slots(shape), experts(shape), shape->fmt) ? 1 : 0;
}

moe_status_t moe_forward(const moe_bf16_t *hidden, const float *logits, const void *w_gu,
                         const void *w_gu_scales, const void *w_d, const void *w_d_scales,
                         const moe_shape_t *shape, moe_bf16_t *out, void *ws, size_t ws_bytes,
                         moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_forward");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!hidden || !logits || !out || !aligned(hidden, 16) || !aligned(out, 16) || !aligned(logits, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_gu, w_gu_scales)) != MOE_OK) return st;
    if ((st = check_weights(shape, w_d, w_d_scales)) != MOE_OK) return st;
    const Layout L = layout(shape, false);
    if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    return forward_device(hidden, logits, w_gu, w_gu_scales, w_d, w_d_scales, shape, out,
                          static_cast<uint8_t *>(ws), L, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward_fused(const moe_bf16_t *hidden, const float *logits, const void *w_gu, const void *w_d,
                               const moe_shape_t *shape, moe_bf16_t *out, void *ws, size_t ws_bytes,
                               moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_forward_fused");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!moe::fused_decode_supported(shape->T, shape->H, shape->I, shape->E, shape->top_k, shape->n_shared,
                                     shape->fmt))
        return MOE_ERR_UNSUPPORTED;
    if (!hidden || !logits || !out || !aligned(hidden, 16) || !aligned(out, 16) || !aligned(logits, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_gu, nullptr)) != MOE_OK) return st;
    if ((st = check_weights(shape, w_d, nullptr)) != MOE_OK) return st;
    const Layout L = layout(shape, false);
    if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    auto *b = static_cast<uint8_t *>(ws);
    return cuda_status(moe::launch_fused_decode(
        logits, hidden, w_gu, w_d, shape->T, shape->H, shape->I, shape->E, shape->top_k, shape->n_shared,
        reinterpret_cast<int32_t *>(b + L.ids), reinterpret_cast<float *>(b + L.w),
        reinterpret_cast<int32_t *>(b + L.counts), reinterpret_cast<int32_t *>(b + L.offsets),
        reinterpret_cast<int32_t *>(b + L.perm), reinterpret_cast<int32_t *>(b + L.inv),
        reinterpret_cast<uint16_t *>(b + L.act), reinterpret_cast<uint16_t *>(b + L.y), out,
        reinterpret_cast<unsigned int *>(b + L.done), error_flag_ptr(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward_host(const moe_bf16_t *hidden_host, const float *logits_host, const void *w_gu,
                              const void *w_gu_scales, const void *w_d, const void *w_d_scales,
                              const moe_shape_t *shape, moe_bf16_t *out_host, void *ws, size_t ws_bytes,
                              moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_forward_host");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!hidden_host || !logits_host || !out_host) return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_gu, w_gu_scales)) != MOE_OK) return st;
    if ((st = check_weights(shape, w_d, w_d_scales)) != MOE_OK) return st;
    const Layout L = layout(shape, true);
    if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    auto *base = static_cast<uint8_t *>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (host_chunks(shape) > 1)
        return forward_host_chunked(hidden_host, logits_host, w_gu, w_gu_scales, w_d, w_d_scales, shape, out_host,
                                    base, L, s);
    const size_t hb = static_cast<size_t>(shape->T) * shape->H * 2;
    const size_t lb = static_cast<size_t>(shape->T) * shape->E * 4;
    if (cudaMemcpyAsync(base + L.hidden_in, hidden_host, hb, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(base + L.logits_in, logits_host, lb, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = forward_device(reinterpret_cast<const moe_bf16_t *>(base + L.hidden_in),
                        reinterpret_cast<const float *>(base + L.logits_in), w_gu, w_gu_scales, w_d, w_d_scales,
                        shape, reinterpret_cast<moe_bf16_t *>(base + L.out_st), base, L, s);
    if (st != MOE_OK) return st;
    if (cudaMemcpyAsync(out_host, base + L.out_st, hb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(s));
}

moe_status_t moe_mx_quantize(const moe_bf16_t *x, int32_t rows, int32_t K, uint8_t *q, uint8_t *scales,
                             moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_mx_quantize");
    if (rows < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
    if (static_cast<long long>(rows) * K >= (1LL << 40)) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!x || !q || !scales || !aligned(x, 16) || !aligned(q, 8)) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_mx_quantize(x, rows, K, q, scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_swiglu_mx(const uint8_t *a_q, const uint8_t *a_scales, const int32_t *perm,
                                        const int32_t *offsets, const void *w_gu, const void *w_gu_scales,
                                        const moe_shape_t *shape, uint8_t *act_q, uint8_t *act_scales,
                                        moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_grouped_gemm_swiglu_mx");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!is_mx(shape->fmt)) return MOE_ERR_INVALID_ARG;
    if (shape->T == 0) return MOE_OK;
    if (!a_q || !a_scales || !offsets || !act_q || !act_scales || !aligned(a_q, 16) || !aligned(a_scales, 4) ||
        !aligned(act_q, 16) || !aligned(offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if (perm && !aligned(perm, 4)) return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_gu, w_gu_scales)) != MOE_OK) return st;
    return cuda_status(moe::launch_grouped_gemm_mxfp8(
        mx_args(shape, a_q, a_scales, perm, offsets, w_gu, w_gu_scales, true, act_q, act_scales, nullptr),
        static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_down_mx(const uint8_t *act_q, const uint8_t *act_scales, const int32_t *offsets,
                                      const void *w_d, const void *w_d_scales, const moe_shape_t *shape,
                                      moe_bf16_t *y, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_grouped_gemm_down_mx");
    moe_status_t st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!is_mx(shape->fmt)) return MOE_ERR_INVALID_ARG;
    if (shape->T == 0) return MOE_OK;
    if (!act_q || !act_scales || !offsets || !y || !aligned(act_q, 16) || !aligned(act_scales, 4) ||
        !aligned(y, 16) || !aligned(offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_weights(shape, w_d, w_d_scales)) != MOE_OK) return st;
    return cuda_status(moe::launch_grouped_gemm_mxfp8(
        mx_args(shape, act_q, act_scales, nullptr, offsets, w_d, w_d_scales, false, nullptr, nullptr, y),
        static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dequant_int4(const uint8_t *q, const moe_bf16_t *scales, int32_t rows, int32_t K,
                              moe_bf16_t *out, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_dequant_int4");
    if (rows < 0 || K <= 0 || K % 128) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!q || !scales || !out || !aligned(q, 16) || !aligned(out, 16) || !aligned(scales, 2))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_dequant_int4(q, scales, rows, K, out, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_device_error(int32_t *code) {
    const moe::NvtxRange nvtx("moe_get_device_error");
    if (!code) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_moe_error_flag, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_moe_error_flag, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    *code = v;
    return MOE_OK;
}

moe_status_t moe_selftest_bounded_wait(int64_t limit_ns, moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_selftest_bounded_wait");
    if (limit_ns < 1 || limit_ns > 1000000000LL) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_bounded_wait_selftest(static_cast<unsigned long long>(limit_ns), error_flag_ptr(),
                                                         static_cast<cudaStream_t>(stream)));
}

const char *moe_status_string(moe_status_t status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or option";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_FLAG: return "device error flag raised";
    }
    return "unknown status";
}

}  // extern "C"
