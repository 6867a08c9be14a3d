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

// Gate activations for callers that pass the gates before their activations
// (Rodimus*, digest.lyk-ai.com summary, "Method": a selection gate g_t, a
// temperature gate tau_t and a low-rank beta_hat_t; the activations are not
// printed, the reading taken is g = softplus(x) = log(1 + e^x), which keeps
// g >= 0, and tau = beta_hat = sigmoid(x) = 1 / (1 + e^-x)).
// Library-accurate versions for the float32 path:
__device__ __forceinline__ float softplus_acc(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_acc(float x) { return 1.0f / (1.0f + expf(-x)); }
// MUFU versions for the bf16 tensor-core path (log1p(y) = y (1 - y/2) to
// ~y^3/3 when y < 1e-3, else log2(1 + y) ln 2; 1 / (1 + inf) = 0 for x -> -inf):
__device__ __forceinline__ float softplus_fast(float x) {
    const float y = ex2_fast(-fabsf(x) * kLog2e);
    const float l = y < 1e-3f ? y * (1.0f - 0.5f * y) : lg2_fast(1.0f + y) * kLn2;
    return fmaxf(x, 0.0f) + l;
}
__device__ __forceinline__ float sigmoid_fast(float x) {
    return __frcp_rn(1.0f + ex2_fast(-x * kLog2e));
}
// g, tau of eight channels in place
__device__ __forceinline__ void activate_gates8(float* g8, float* t8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        g8[e] = softplus_fast(g8[e]);
        t8[e] = sigmoid_fast(t8[e]);
    }
}
// beta_hat = sigmoid(x) = (1 + tanh(x / 2)) / 2 with the single-instruction
// tanh (PTX tanh.approx, relative error about 2^-11): beta_hat only scales v,
// whose bf16 rounding (2^-9) already bounds the path's accuracy, so one MUFU
// operation per element replaces the exponential and the reciprocal.  (tau
// keeps sigmoid_fast: its errors compound along the decay products.)
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sigmoid_tanh(float x) { return fmaf(0.5f, tanh_fast(0.5f * x), 0.5f); }
__device__ __forceinline__ void activate_beta8(float* b8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) b8[e] = sigmoid_tanh(b8[e]);
}

// Device status word bits (set with atomicOr by kernels, read by the host).
constexpr unsigned kErrTimeout = 1u;

}  // namespace rdm
