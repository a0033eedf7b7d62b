// common.cuh -- small helpers shared by the MoE kernels and their launchers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "../../include/moe.h"

namespace moe {

// Device status word kept at the start of a workspace.  0 = fine; otherwise
// kDeviceTimeoutBase | role of the first wait that gave up.
constexpr int kDeviceTimeoutBase = 0x100;
constexpr int kRoleProducer = 1;
constexpr int kRoleMma = 2;
constexpr int kRoleEpilogue = 3;
constexpr int kRoleTest = 4;

// Default bound on any device-side wait: far above the longest legitimate wait
// (one tile of the longest contraction, tens of microseconds).
constexpr uint64_t kDefaultWaitTimeoutNs = 2000000000ull;

constexpr size_t kWsHeaderBytes = 256;  // status word + scheduling state

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) {
    return (v + a - 1) / a * a;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even, lo in the low half
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Host side --------------------------------------------------------------------
int device_sm_count();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Programmatic dependent launch.  The layer's kernels are launched with
// programmatic stream serialisation: a kernel's CTAs may be scheduled as the
// previous kernel's CTAs exit, and run their prologue (barrier set-up,
// tensor-memory allocation, descriptor prefetch) during its tail.  Every such
// kernel calls grid_dependency_wait() unconditionally, before it reads anything
// the previous kernel wrote and before any early exit: it returns once the
// previous grid has completed and its memory operations are visible, so
// completion of a kernel still implies completion of everything before it in
// the stream.  Launched without the attribute, the wait returns at once.  No
// kernel triggers its dependents early (griddepcontrol.launch_dependents):
// waiting CTAs of the next kernel then sat on the SMs during the whole launch,
// which measured slower at T = 4096.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Raises `kernel`'s dynamic shared-memory limit to at least `bytes` on the
// current device, calling the runtime only the first time (or when more is
// needed): keeps the per-launch host path free of attribute calls, which also
// keeps it legal inside stream capture.
inline bool ensure_dynamic_smem(const void* kernel, int bytes) {
    struct Entry {
        const void* kernel;
        int device;
        int bytes;
    };
    static std::mutex mu;
    static Entry cache[128];
    static int n = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i) {
        if (cache[i].kernel != kernel || cache[i].device != dev) continue;
        if (cache[i].bytes >= bytes) return true;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
            return false;
        cache[i].bytes = bytes;
        return true;
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    if (n < 128) cache[n++] = Entry{kernel, dev, bytes};
    return true;
}

// kernel<<<grid, block, smem, stream>>>(args...) with programmatic stream
// serialisation allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
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
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
