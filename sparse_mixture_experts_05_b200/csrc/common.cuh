// common.cuh -- small helpers shared by the MoE kernels and their launchers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

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

}  // namespace moe
