// Shared helpers of the CUDA library (device utilities, status words, host checks).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------------------
// host-side argument checks
// ---------------------------------------------------------------------------
#define MOE_REQUIRE(cond, code)     \
    do {                            \
        if (!(cond)) return (code); \
    } while (0)

#define MOE_CUDA_TRY(expr)                          \
    do {                                            \
        cudaError_t err_ = (expr);                  \
        if (err_ != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// Checks that the last kernel launch was accepted.
inline int launch_status() {
    return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t dtype_size(moe_dtype d) { return d == MOE_BF16 ? 2 : 4; }

inline bool valid_dtype(int d) { return d == MOE_F32 || d == MOE_BF16; }

// Number of SMs and other per-device facts, cached per device.
int device_sm_count();

// ---------------------------------------------------------------------------
// device-side status word: first error wins, never cleared by a kernel
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Upper bound on any single wait inside a kernel, in nanoseconds.  A wait that
// exceeds it reports MOE_ERR_TIMEOUT and the kernel winds down.
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// ---------------------------------------------------------------------------
// element loads/stores in either supported dtype
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe
