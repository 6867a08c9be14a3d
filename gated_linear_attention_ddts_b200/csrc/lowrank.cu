// lowrank.cu -- the low-rank beta_hat of the Rodimus block (Rodimus*,
// digest.lyk-ai.com summary, "Method": beta_hat is built from low-rank
// matrices, which cuts parameters and filters input noise).  This library's
// reading: a per-token factor u [B,T,r], shared by the heads (the token's input
// projected down to rank r by the layer), times an up-projection w_up
// [H,r,d_v] gives beta_hat's pre-activation
//
//   beta_pre[b,h,t,j] = sum_rho u[b,t,rho] w_up[h,rho,j],   beta_hat = sigmoid(beta_pre)
//
// The forward builds it on chip inside the tensor-core kernel.  The backward
// runs the pre-activation backward on an expanded copy and contracts its
// gradient db = dL/dbeta_pre:
//
//   du[b,t,rho]    = sum_{h,j} db[b,h,t,j] w_up[h,rho,j]
//   dw_up[h,rho,j] = sum_{b,t} u[b,t,rho] db[b,h,t,j]
//
// These three kernels are plain streaming loops on the CUDA cores (r <= 16).
#include "launch.h"
#include "rdm_common.cuh"

namespace rdm {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float ld(const T* p) { return ldf(p); }

// one thread per (b, h, t, 8 channels): beta_pre written in the sequence dtype
template <typename T>
__global__ void __launch_bounds__(kThreads) lr_expand_kernel(const LowRankParams p) {
    const int J8 = p.dv / 8;
    const long long n = (long long)p.B * p.H * p.T * J8;
    for (long long i = blockIdx.x * (long long)kThreads + threadIdx.x; i < n;
         i += (long long)gridDim.x * kThreads) {
        const int j8 = (int)(i % J8);
        const long long row = i / J8;  // (b*H + h)*T + t
        const int t = (int)(row % p.T);
        const long long bh = row / p.T;
        const int h = (int)(bh % p.H), b = (int)(bh / p.H);
        const T* u = static_cast<const T*>(p.u) + ((size_t)b * p.T + t) * p.r;
        const float* w = p.w + (size_t)h * p.r * p.dv + j8 * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int rho = 0; rho < p.r; ++rho) {
            const float ur = ld(u + rho);
            const float4 wa = __ldg(reinterpret_cast<const float4*>(w + (size_t)rho * p.dv));
            const float4 wb = __ldg(reinterpret_cast<const float4*>(w + (size_t)rho * p.dv + 4));
            acc[0] = fmaf(ur, wa.x, acc[0]); acc[1] = fmaf(ur, wa.y, acc[1]);
            acc[2] = fmaf(ur, wa.z, acc[2]); acc[3] = fmaf(ur, wa.w, acc[3]);
            acc[4] = fmaf(ur, wb.x, acc[4]); acc[5] = fmaf(ur, wb.y, acc[5]);
            acc[6] = fmaf(ur, wb.z, acc[6]); acc[7] = fmaf(ur, wb.w, acc[7]);
        }
        T* out = static_cast<T*>(p.beta_pre) + (size_t)row * p.dv + j8 * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) stf(out + e, acc[e]);
    }
}

// du: one thread per (b, t, rho); the r threads of a token read the same db
// rows (broadcast through L1), w_up stays in L1/L2
template <typename T>
__global__ void __launch_bounds__(kThreads) lr_grad_u_kernel(const LowRankParams p) {
    const long long n = (long long)p.B * p.T * p.r;
    for (long long i = blockIdx.x * (long long)kThreads + threadIdx.x; i < n;
         i += (long long)gridDim.x * kThreads) {
        const int rho = (int)(i % p.r);
        const long long bt = i / p.r;
        const int t = (int)(bt % p.T), b = (int)(bt / p.T);
        float acc = 0.0f;
        for (int h = 0; h < p.H; ++h) {
            const T* db = static_cast<const T*>(p.dbeta_pre) + (((size_t)b * p.H + h) * p.T + t) * p.dv;
            const float* w = p.w + ((size_t)h * p.r + rho) * p.dv;
            for (int j = 0; j < p.dv; ++j) acc = fmaf(ld(db + j), __ldg(w + j), acc);
        }
        stf(static_cast<T*>(p.du) + i, acc);
    }
}

// dw_up: block (h, token range); thread (rho, 8 channels) sums over the range,
// then one float32 atomic per value and block (dw_up zeroed beforehand)
template <typename T>
__global__ void __launch_bounds__(kThreads) lr_grad_w_kernel(const LowRankParams p, int tokens_per_block) {
    const int h = blockIdx.y;
    const int J8 = p.dv / 8;
    const long long BT = (long long)p.B * p.T;
    const long long s0 = (long long)blockIdx.x * tokens_per_block;
    const long long s1 = s0 + tokens_per_block < BT ? s0 + tokens_per_block : BT;
    for (int k = threadIdx.x; k < p.r * J8; k += kThreads) {
        const int rho = k / J8, j8 = k % J8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (long long bt = s0; bt < s1; ++bt) {
            const int t = (int)(bt % p.T), b = (int)(bt / p.T);
            const float ur = ld(static_cast<const T*>(p.u) + bt * p.r + rho);
            const T* db = static_cast<const T*>(p.dbeta_pre) + (((size_t)b * p.H + h) * p.T + t) * p.dv + j8 * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(ur, ld(db + e), acc[e]);
        }
        float* dw = p.dw + ((size_t)h * p.r + rho) * p.dv + j8 * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) atomicAdd(dw + e, acc[e]);
    }
}

unsigned grid_for(long long n) {
    const long long b = (n + kThreads - 1) / kThreads;
    return (unsigned)(b < 1 ? 1 : (b > 148LL * 16 ? 148LL * 16 : b));
}

}  // namespace

cudaError_t launch_lowrank_expand(const LowRankParams& p, cudaStream_t s) {
    const long long n = (long long)p.B * p.H * p.T * (p.dv / 8);
    if (p.bf16) lr_expand_kernel<__nv_bfloat16><<<grid_for(n), kThreads, 0, s>>>(p);
    else lr_expand_kernel<float><<<grid_for(n), kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_grad(const LowRankParams& p, cudaStream_t s) {
    const long long nu = (long long)p.B * p.T * p.r;
    if (p.bf16) lr_grad_u_kernel<__nv_bfloat16><<<grid_for(nu), kThreads, 0, s>>>(p);
    else lr_grad_u_kernel<float><<<grid_for(nu), kThreads, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p.dw, 0, (size_t)p.H * p.r * p.dv * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const long long BT = (long long)p.B * p.T;
    // about four blocks per SM over all heads
    long long per = (BT * p.H + 4 * 148 - 1) / (4 * 148);
    per = per < 64 ? 64 : per;
    const unsigned gx = (unsigned)((BT + per - 1) / per);
    const dim3 grid(gx < 1 ? 1 : gx, (unsigned)p.H);
    if (p.bf16) lr_grad_w_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p, (int)per);
    else lr_grad_w_kernel<float><<<grid, kThreads, 0, s>>>(p, (int)per);
    return cudaGetLastError();
}

}  // namespace rdm
