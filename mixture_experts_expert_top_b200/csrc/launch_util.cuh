// launch_util.cuh -- kernel launches with programmatic dependent launch.
//
// Every kernel of libmoe_b200 is launched with programmatic stream
// serialization, so it may start while the previous kernel on the stream is
// still finishing. Each kernel first does set-up that reads nothing written
// on the stream (barrier init, TMEM allocation, tensor-map prefetch), then
// calls griddep_wait(), which returns once the previous grid has completed
// and its writes are visible; only then does it read its inputs.
// griddep_launch_dependents() lets the next kernel be scheduled once every CTA
// of this one has called it (or exited). The small routing and bucketing
// kernels call it at once, so that the GEMM behind them sets up on the idle
// SMs; the GEMMs call it only when all their roles are done, because CTAs of
// the next kernel that share an SM with a running GEMM CTA slow it down; the
// combine kernel never calls it (exit is the trigger).
#pragma once

#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

namespace moe {

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel, device and
// size: it is a driver call that would otherwise run on every launch.
template <typename... KArgs>
inline cudaError_t ensure_dynamic_smem(void (*kernel)(KArgs...), size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = 0;
    cudaError_t st = cudaGetDevice(&dev);
    if (st != cudaSuccess) return st;
    const auto key = std::make_pair(reinterpret_cast<const void *>(kernel), dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    st = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (st == cudaSuccess) done[key] = bytes;
    return st;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
