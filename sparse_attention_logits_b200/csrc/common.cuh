// Shared device/host helpers of the sm_100a DSA library (no kernels here).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/dsa_b200.h"

namespace dsa {

// Device error word codes (bit flags), written by kernels that give up a
// bounded wait.  Read and cleared by dsa_get_device_error().
enum : unsigned {
    DEV_ERR_NONE = 0u,
    DEV_ERR_TIMEOUT_TMA = 1u,      // a wait for a bulk/tensor copy ran out
    DEV_ERR_TIMEOUT_MMA = 2u,      // a wait for a tensor-core commit ran out
    DEV_ERR_TIMEOUT_PEER = 4u,     // a wait on a partner CTA of the cluster ran out
    DEV_ERR_BAD_INDEX = 8u,        // an index outside [0, ctx_len) was met and skipped
};

constexpr int kMaxDevices = 64;

// Lock held while a per-device value is computed for the first time (the
// device error word's address, occupancy queries); later calls read the
// published value without it.
std::mutex& init_mutex();

// Per-device integer computed on first use: 0 = not yet known.  The first
// callers on a device run `compute` under init_mutex(); its result (or -1
// when it gives no positive value) is then published.  Returns the cached
// value, or 0 when there is none.
template <class F>
int device_cached(std::atomic<int> (&cache)[kMaxDevices], F&& compute) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    int v = cache[dev].load(std::memory_order_acquire);
    if (v == 0) {
        std::lock_guard<std::mutex> lock(init_mutex());
        v = cache[dev].load(std::memory_order_relaxed);
        if (v == 0) {
            const int n = compute();
            v = n > 0 ? n : -1;
            cache[dev].store(v, std::memory_order_release);
        }
    }
    return v > 0 ? v : 0;
}

struct Launch {
    cudaStream_t stream;
    unsigned* err;   // device error word of the current device
    int num_sms;
};

// Per-thread count of kernel launches (exported as dsa_launch_count()).
void count_launch(int n = 1);

__device__ __forceinline__ void record_error(unsigned* err, unsigned code) {
    if (err) atomicOr(err, code);
}

template <typename T> struct ElemTraits;
template <> struct ElemTraits<float> {
    static __device__ __forceinline__ float to_f32(float v) { return v; }
};
template <> struct ElemTraits<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
};
template <> struct ElemTraits<__nv_fp8_e4m3> {
    static __device__ __forceinline__ float to_f32(__nv_fp8_e4m3 v) { return float(v); }
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__nv_fp8_e4m3 v) { return float(v); }

__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Order-preserving map of an fp32 score to uint32 (larger score -> larger
// key); -0.0 is first made +0.0 so that the two zeros tie.
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch.  The step's kernels are launched with the
// programmatic-serialisation attribute, so the next kernel of the stream may
// be scheduled while this one drains.  pdl_wait() blocks until every kernel
// the grid depends on has completed and its writes are visible (a no-op when
// launched without the attribute): nothing before it may read or write global
// memory that another kernel touches.  pdl_launch_dependents() lets the next
// kernel's CTAs start (they too wait before touching memory).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
inline cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

}  // namespace dsa
