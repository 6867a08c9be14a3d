// rdm_common.cuh -- device helpers shared by the DDTS kernels: element
// load/store for float32 / bf16, the DDTS gate formulas, and the launcher
// parameter blocks.  Gates follow the DDTS definition of Rodimus* (digest.lyk-ai.com
// summary, "Method"): alpha = exp(-g*tau), alpha_hat = g^tau.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rdm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float* p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// log(alpha) = -g*tau, in natural-log units.
__device__ __forceinline__ float log_alpha(float g, float tau) { return -g * tau; }

// log2(alpha_hat) = tau * log2(g), with the power conventions 0^0 = 1 (tau == 0
// gives 0 for every g) and 0^tau = 0 for tau > 0 (log2(0) = -inf).
__device__ __forceinline__ float log2_alpha_hat(float g, float tau) {
    return tau == 0.0f ? 0.0f : tau * log2f(g);
}

__device__ __forceinline__ float alpha_hat(float g, float tau) {
    return exp2f(log2_alpha_hat(g, tau));
}

__device__ __forceinline__ float alpha(float g, float tau) {
    return exp2f(log_alpha(g, tau) * kLog2e);
}

// Single MUFU instructions (PTX ex2.approx / lg2.approx, flush-to-zero): 2^x
// and log2(x) to about 22 bits, with ex2(-inf) = 0 and lg2(0) = -inf.  Used on
// the bf16 tensor-core path, where every result is rounded to 8 bits anyway.
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Device status word bits (set with atomicOr by kernels, read by the host).
constexpr unsigned kErrTimeout = 1u;

}  // namespace rdm
