// noalloc.cu -- moe_permute_noalloc: the permute (bucketing) step for callers
// that cannot allocate device memory.
//
// moe_permute needs scratch (a per-chunk expert histogram) once a call has
// more than 8192 (token, expert) pairs, and asks its caller for it. Some
// callers cannot hand out device memory: code that runs as a plugin of a host
// framework which owns every device allocation and passes no workspace, and
// code whose hot loop must never call cudaMalloc because that call can
// synchronise the device and stall other work on it. This entry point takes
// the same scratch from a fixed array compiled into the library instead.
//
// The array lives in this file, in device memory of every GPU that loads the
// library, until the process exits. Its device address is looked up once per
// device, on the first call made with that device current.
#include <stdint.h>

#include <atomic>

#include "launch.h"
#include "moe.h"

namespace {

// Largest chunk histogram the array holds: nchunks * E int32 entries, where
// nchunks = ceil(T*top_k / 2048) once T*top_k > 8192. 65536 entries = 256 KiB.
constexpr int kScratchInts = 65536;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

// Device address of g_permute_scratch on the current device (nullptr on
// failure). In host code the symbol's name is only a host-side stand-in, so
// the address has to come from cudaGetSymbolAddress with the device current.
// Concurrent first calls on one device may both look it up; they store the
// same address. The address belongs to the device's context, so it is not
// valid across a cudaDeviceReset.
int32_t *scratch_ptr() {
    static std::atomic<int32_t *> ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int32_t *p = ptrs[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_permute_scratch) != cudaSuccess) return nullptr;
        ptrs[dev].store(p, std::memory_order_release);
    }
    return p;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const int32_t *topk_ids, const moe_shape_t *shape, int32_t *counts,
                                            int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                            const moe_bf16_t *hidden, moe_bf16_t *hidden_perm,
                                            moe_stream_t stream) {
    const moe::NvtxRange nvtx("moe_permute_noalloc");
    // the same argument rules as moe_permute
    const moe_status_t st = moe::validate_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    const long long P = static_cast<long long>(shape->T) * moe::shape_slots(shape);
    const int E = moe::shape_experts(shape);
    if (!counts || !offsets || !topk_ids || !perm || !inv_perm || !aligned(counts, 4) || !aligned(offsets, 4) ||
        !aligned(topk_ids, 4) || !aligned(perm, 4) || !aligned(inv_perm, 4))
        return MOE_ERR_INVALID_ARG;
    if ((hidden == nullptr) != (hidden_perm == nullptr)) return MOE_ERR_INVALID_ARG;
    if (hidden && (!aligned(hidden, 16) || !aligned(hidden_perm, 16))) return MOE_ERR_INVALID_ARG;
    // the chunk histogram must fit the built-in array
    if (moe::permute_scratch_bytes(P, E) > sizeof(int32_t) * static_cast<size_t>(kScratchInts))
        return MOE_ERR_UNSUPPORTED;
    int32_t *scratch = scratch_ptr();
    if (!scratch) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = moe::launch_permute(topk_ids, static_cast<int>(P), E, counts, offsets, perm, inv_perm,
                                        scratch, moe::device_error_flag(), s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (hidden)
        e = moe::launch_gather(hidden, perm, static_cast<int>(P), shape->H, moe::shape_slots(shape), hidden_perm,
                               moe::device_error_flag(), s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
