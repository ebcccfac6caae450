// common.cuh -- device helpers shared by the RG-LRU kernels (math, dtype conversion, status).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rglru.h"

#include <mutex>

namespace rglru {

// Unique id of the calling thread's current CUDA context (0 when unavailable).
unsigned long long current_context_id();

// Sets a kernel's dynamic shared-memory limit once per kernel and context (the attribute belongs
// to the kernel in the current context; doing it on the first call keeps it out of any later
// stream capture, and a new context -- after a cudaDeviceReset -- gets it again).
cudaError_t set_smem_limit(const void* kernel, int bytes);

template <typename Kernel>
cudaError_t set_smem_once(Kernel k, int bytes) {
    return set_smem_limit(reinterpret_cast<const void*>(k), bytes);
}

constexpr int kConvWidth = 4;
constexpr int kHist = kConvWidth - 1;

// Device status word at the start of every workspace (first 16 bytes).
struct DeviceStatus {
    unsigned int code;     // rglru_status latched by the first failing CTA (0 = OK)
    unsigned int where;    // kernel-specific location of the failure
    unsigned int info0;
    unsigned int info1;
};

__device__ __forceinline__ void latch_status(DeviceStatus* st, unsigned code, unsigned where,
                                             unsigned info0, unsigned info1) {
    if (st && atomicCAS(&st->code, 0u, code) == 0u) {
        st->where = where;
        st->info0 = info0;
        st->info1 = info1;
    }
}

// ---- element access for the two activation dtypes --------------------------------------
template <typename T> struct Act;
template <> struct Act<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Act<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// ---- accurate fp32 math (CUDA's own libdevice functions, no fast-math) --------------------
// sigma(z) = 1 / (1 + e^{-z}); for z -> -inf, expf overflows to inf and the result is 0.
__device__ __forceinline__ float sigmoid_acc(float z) { return 1.0f / (1.0f + expf(-z)); }
// log sigma(z) = -softplus(-z) = min(z, 0) - log1p(e^{-|z|})
__device__ __forceinline__ float log_sigmoid_acc(float z) {
    return fminf(z, 0.0f) - log1pf(expf(-fabsf(z)));
}
// v * Phi(v) = 0.5 v erfc(-v / sqrt 2) (no cancellation for v << 0)
__device__ __forceinline__ float gelu_exact_acc(float v) {
    return 0.5f * v * erfcf(-v * 0.70710678118654752440f);
}
// 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))
__device__ __forceinline__ float gelu_tanh_acc(float v) {
    const float k = 0.79788456080286535588f;
    return 0.5f * v * (1.0f + tanhf(k * (v + 0.044715f * v * v * v)));
}
__device__ __forceinline__ float gelu_acc(float v, int tanh_form) {
    return tanh_form ? gelu_tanh_acc(v) : gelu_exact_acc(v);
}

// Decay and input normalisation of one element: log a = c r log sigma(Lambda) (<= 0),
// a = e^{log a}, beta = sqrt(1 - a^2) = sqrt(-expm1(2 log a)) (exact near a = 1).
__device__ __forceinline__ void decay_and_beta_acc(float c_log_a_base, float r, float* a,
                                                   float* beta) {
    float la = c_log_a_base * r;
    *a = expf(la);
    *beta = sqrtf(-expm1f(2.0f * la));
}

}  // namespace rglru
