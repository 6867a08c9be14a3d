// feed.cu -- gradient of the feedthrough weights d of o_t += d (.) v_t.
//
// The pages name the feedthrough d_t of Eq. (11) as the SSM feedthrough term
// (paperhub.cn OpenReview rebuttal, answer to Q6: the design Mamba and Mamba2
// use, a learned per-channel skip from the SSM input to its output); the
// forward adds it in the store stage of the output and the backward adds
// d (.) dO_t to dv in its dv epilogue.  What remains is the weight gradient,
// a reduction over batch and time per (head, value channel):
//     grad_d[h][j] = sum_{b,t} dO[b,h,t,j] * v[b,h,t,j]
// One block per (b,h) and tile of tokens; columns across threads (coalesced
// rows), tokens strided over the rest of the block, a shared-memory reduction
// over the token lanes, then one float32 atomic per column and block.
#include "launch.h"
#include "rdm_common.cuh"

namespace rdm {
namespace {

constexpr int kThreads = 256;
constexpr int kTileT = 512;  // tokens per block

template <typename T>
__global__ void __launch_bounds__(kThreads) feed_grad_kernel(BwdParams p) {
    const int bh = blockIdx.x, h = bh % p.H;
    const int dv = p.dv, rows = kThreads / dv;  // dv divides 256 (16..128)
    const int j = threadIdx.x % dv, r = threadIdx.x / dv;
    const int t0 = blockIdx.y * kTileT, t1 = min(p.T, t0 + kTileT);
    const T* dO = static_cast<const T*>(p.dO) + (size_t)bh * p.T * dv;
    const T* v = static_cast<const T*>(p.v) + (size_t)bh * p.T * dv;
    float acc = 0.0f;
    for (int t = t0 + r; t < t1; t += rows) acc = fmaf(ldf(dO + (size_t)t * dv + j), ldf(v + (size_t)t * dv + j), acc);
    __shared__ float red[kThreads];
    red[threadIdx.x] = acc;
    __syncthreads();
    if (r == 0) {
        for (int k = 1; k < rows; ++k) acc += red[k * dv + j];
        atomicAdd(p.grad_dfeed + (size_t)h * dv + j, acc);
    }
}

}  // namespace

cudaError_t launch_feed_grad(const BwdParams& p, cudaStream_t s) {
    if (!p.grad_dfeed) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(p.grad_dfeed, 0, (size_t)p.H * p.dv * sizeof(float), s);
    if (e != cudaSuccess || p.T == 0 || p.B * p.H == 0) return e;
    const dim3 grid(p.B * p.H, (p.T + kTileT - 1) / kTileT);
    if (p.bf16)
        feed_grad_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p);
    else
        feed_grad_kernel<float><<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace rdm
