// shortconv.cu -- the ShortConv of the Rodimus block: a causal depthwise
// convolution along the tokens (digest.lyk-ai.com summary of Rodimus*,
// "Method", third Rodimus bullet: a short convolution for local context next
// to the GLU; width, activation and carried state are this library's reading):
//
//   z[b,h,t,c] = bias[h,c] + sum_{i<W} w[h,c,i] x[b,h,t-i,c],   y = z or z*sigmoid(z)
//
// with x at t-i < 0 read from the carried-in state (the previous W-1 inputs).
//
// HBM-bound streaming: one thread owns 16 bytes of channels (8 bf16 or 4
// float32) over a run of kRun consecutive tokens and keeps the last W inputs
// of its channels in registers, so every input row is read once per run (plus
// a W-1 row halo that the neighbouring run of the same block has just pulled
// into L1) and every output row written once; a warp's loads and stores cover
// whole 16-byte column groups of consecutive rows.  Runs are short and fully
// unrolled so that each thread has all of its loads in flight at once (with
// 16-token runs walked one load at a time the kernels ran at 7% of HBM).  The backward walks the same runs with a
// look-ahead window of W values of dL/dz, and reduces the weight and bias
// gradients in shared memory before one float32 atomic per value and block.
#include <algorithm>

#include "launch.h"
#include "rdm_common.cuh"

namespace rdm {
namespace {

constexpr int kThreads = 256;
constexpr int kRun = 4;  // tokens per thread (loops fully unrolled: every load in flight at once)

template <typename T>
struct Vec {
    static constexpr int N = 16 / sizeof(T);  // channels per 16-byte group
};

// inputs are read through the read-only path (x, dy and the states are never
// written by these kernels; the API requires outputs not to alias inputs), so
// the loads of a run can be issued ahead of its stores
__device__ __forceinline__ void load_vec(const float* p, float* f) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float* f) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ void store_vec(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    *reinterpret_cast<uint4*>(p) = u;
}

// input row t (t < 0: from the carried-in state, zeros without one) of my channels
template <typename T>
__device__ __forceinline__ void input_row(const ConvParams& p, int bh, int t, int c0, float* f) {
    constexpr int N = Vec<T>::N;
    if (t >= 0 && t < p.T) {
        load_vec(static_cast<const T*>(p.x) + ((size_t)bh * p.T + t) * p.D + c0, f);
    } else if (t < 0 && p.xs != nullptr && p.W - 1 + t >= 0) {
        load_vec(static_cast<const T*>(p.xs) + ((size_t)bh * (p.W - 1) + (p.W - 1 + t)) * p.D + c0, f);
    } else {
#pragma unroll
        for (int e = 0; e < N; ++e) f[e] = 0.0f;
    }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }
// d silu / dz = s (1 + z (1 - s)), s = sigmoid(z)
__device__ __forceinline__ float silu_grad(float z) {
    const float s = 1.0f / (1.0f + __expf(-z));
    return s * (1.0f + z * (1.0f - s));
}

template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv_fwd_kernel(ConvParams p) {
    constexpr int N = Vec<T>::N;
    const int CG = p.D / N, R = kThreads / CG;
    const int bh = blockIdx.x, h = bh % p.H;
    const int cg = threadIdx.x % CG, run = threadIdx.x / CG, c0 = cg * N;
    const int t0 = (blockIdx.y * R + run) * kRun, t1 = min(t0 + kRun, p.T);
    if (t0 >= p.T) return;  // no barrier in this kernel
    float wv[W][N], bv[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i < W; ++i) wv[i][e] = p.w[((size_t)h * p.D + c0 + e) * W + i];
        bv[e] = p.bias ? p.bias[(size_t)h * p.D + c0 + e] : 0.0f;
    }
    float win[W][N];  // win[k] = x[t - (W-1) + k]
#pragma unroll
    for (int k = 0; k < W - 1; ++k) input_row<T>(p, bh, t0 - (W - 1) + k, c0, win[k]);
    T* y = static_cast<T*>(p.y) + (size_t)bh * p.T * p.D + c0;
#pragma unroll
    for (int k = 0; k < kRun; ++k) {
        const int t = t0 + k;
        if (t >= t1) break;
        input_row<T>(p, bh, t, c0, win[W - 1]);
        float z[N];
#pragma unroll
        for (int e = 0; e < N; ++e) {
            float a = bv[e];
#pragma unroll
            for (int i = 0; i < W; ++i) a = fmaf(wv[i][e], win[W - 1 - i][e], a);
            z[e] = p.silu ? silu_f(a) : a;
        }
        store_vec(y + (size_t)t * p.D, z);
#pragma unroll
        for (int k = 0; k < W - 1; ++k)
#pragma unroll
            for (int e = 0; e < N; ++e) win[k][e] = win[k + 1][e];
    }
}

// state after the sequence: its last W-1 inputs (carried-in ones when T < W-1)
template <typename T>
__global__ void conv_state_kernel(ConvParams p) {
    const size_t n = (size_t)p.B * p.H * (p.W - 1) * p.D;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % p.D), s = (int)((idx / p.D) % (p.W - 1));
        const size_t bh = idx / ((size_t)p.D * (p.W - 1));
        const int t = p.T - (p.W - 1) + s;
        float v = 0.0f;
        if (t >= 0) v = ldf(static_cast<const T*>(p.x) + (bh * p.T + t) * p.D + c);
        else if (p.xs) v = ldf(static_cast<const T*>(p.xs) + (bh * (p.W - 1) + (p.W - 1 + t)) * p.D + c);
        stf(static_cast<T*>(p.xs_out) + idx, v);
    }
}

// dL/dz at token t (zero past the end): dy, through the SiLU when on
template <typename T, int W>
__device__ __forceinline__ void dz_row(const ConvParams& p, int bh, int t, int c0, const float (&wv)[W][Vec<T>::N],
                                       const float* bv, float* dz) {
    constexpr int N = Vec<T>::N;
    if (t >= p.T) {
#pragma unroll
        for (int e = 0; e < N; ++e) dz[e] = 0.0f;
        return;
    }
    load_vec(static_cast<const T*>(p.dy) + ((size_t)bh * p.T + t) * p.D + c0, dz);
    if (p.silu) {
        float xw[W][N];
#pragma unroll
        for (int i = 0; i < W; ++i) input_row<T>(p, bh, t - i, c0, xw[i]);
#pragma unroll
        for (int e = 0; e < N; ++e) {
            float a = bv[e];
#pragma unroll
            for (int i = 0; i < W; ++i) a = fmaf(wv[i][e], xw[i][e], a);
            dz[e] *= silu_grad(a);
        }
    }
}

template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv_bwd_kernel(ConvParams p) {
    constexpr int N = Vec<T>::N;
    const int CG = p.D / N, R = kThreads / CG;
    const int bh = blockIdx.x, h = bh % p.H;
    const int cg = threadIdx.x % CG, run = threadIdx.x / CG, c0 = cg * N;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // per-warp partial sums of the weight and bias gradients: [warp][cg][W+1][N]
    __shared__ float s_red[kThreads / 32][128 * 5];  // CG (W + 1) N = D (W + 1) <= 640
    float wv[W][N], bv[N], aw[W][N], ab[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i < W; ++i) {
            wv[i][e] = p.w[((size_t)h * p.D + c0 + e) * W + i];
            aw[i][e] = 0.0f;
        }
        bv[e] = p.bias ? p.bias[(size_t)h * p.D + c0 + e] : 0.0f;
        ab[e] = 0.0f;
    }
    T* dx = static_cast<T*>(p.dx) + (size_t)bh * p.T * p.D + c0;
    const int tout0 = p.T - (p.W - 1);  // first token copied into the carried-out state
    // the block's tile of tokens is a whole number of R x kRun groups; every
    // thread walks its run in each group (the weight gradients accumulate in
    // registers across the groups)
    for (int t0 = (blockIdx.y * p.conv_groups * R + run) * kRun; t0 < min(p.T, (blockIdx.y + 1) * p.conv_groups * R * kRun);
         t0 += R * kRun) {
        const int t1 = min(t0 + kRun, p.T);
        // dzw[k] = dz[t + k] for the output t = the oldest token of the window
        float dzw[W][N];
#pragma unroll
        for (int k = 0; k < W - 1; ++k) dz_row<T, W>(p, bh, t0 + k, c0, wv, bv, dzw[k]);
#pragma unroll
        for (int k = 0; k < kRun; ++k) {
            const int t = t0 + k;
            if (t >= t1) break;
            dz_row<T, W>(p, bh, t + W - 1, c0, wv, bv, dzw[W - 1]);
            float xw[W][N];  // x[t - i]
#pragma unroll
            for (int i = 0; i < W; ++i) input_row<T>(p, bh, t - i, c0, xw[i]);
            float g[N];
#pragma unroll
            for (int e = 0; e < N; ++e) {
                float a = 0.0f;
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    a = fmaf(wv[i][e], dzw[i][e], a);                // dx[t] = sum_i w_i dz[t + i]
                    aw[i][e] = fmaf(dzw[0][e], xw[i][e], aw[i][e]);  // dw_i += dz[t] x[t - i]
                }
                ab[e] += dzw[0][e];
                g[e] = a;
            }
            if (p.dxs_out != nullptr && t >= tout0) {  // the carried-out state copies x[t]
                float go[N];
                load_vec(static_cast<const T*>(p.dxs_out) + ((size_t)bh * (p.W - 1) + (t - tout0)) * p.D + c0, go);
#pragma unroll
                for (int e = 0; e < N; ++e) g[e] += go[e];
            }
            store_vec(dx + (size_t)t * p.D, g);
#pragma unroll
            for (int kk = 0; kk < W - 1; ++kk)
#pragma unroll
                for (int e = 0; e < N; ++e) dzw[kk][e] = dzw[kk + 1][e];
        }
    }
    // weight and bias gradients: sum the lanes of a warp that hold the same
    // channels (lanes cg, cg + CG, ...), one slot per warp in shared memory, a
    // sum over the warps, then one float32 atomic per value and block
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i <= W; ++i) {
            float x = i < W ? aw[i][e] : ab[e];
            for (int off = CG; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (lane < CG) s_red[warp][(cg * (W + 1) + i) * N + e] = x;
        }
    }
    __syncthreads();
    // CG divides 32, so every warp holds every channel group
    for (int idx = threadIdx.x; idx < CG * (W + 1) * N; idx += kThreads) {
        const int e = idx % N, i = (idx / N) % (W + 1), gi = idx / (N * (W + 1));
        float a = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < kThreads / 32; ++w2) a += s_red[w2][idx];
        const int c = gi * N + e;
        if (i < W) atomicAdd(p.dw + ((size_t)h * p.D + c) * W + i, a);
        else if (p.dbias) atomicAdd(p.dbias + (size_t)h * p.D + c, a);
    }
    (void)R;
}

// gradient of the carried-in state: dxs[s] = sum_i w_i dz[s-(W-1)+i] over tokens
// 0..T-1, plus the carried-out state's gradient where it copies a carried-in
// input (T < W-1)
template <typename T, int W>
__global__ void conv_state_grad_kernel(ConvParams p) {
    constexpr int N = Vec<T>::N;
    const int CG = p.D / N;
    const size_t n = (size_t)p.B * p.H * (W - 1) * CG;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int cg = (int)(idx % CG), s = (int)((idx / CG) % (W - 1));
        const int bh = (int)(idx / ((size_t)CG * (W - 1))), h = bh % p.H, c0 = cg * N;
        float wv[W][N], bv[N], g[N];
#pragma unroll
        for (int e = 0; e < N; ++e) {
#pragma unroll
            for (int i = 0; i < W; ++i) wv[i][e] = p.w[((size_t)h * p.D + c0 + e) * W + i];
            bv[e] = p.bias ? p.bias[(size_t)h * p.D + c0 + e] : 0.0f;
            g[e] = 0.0f;
        }
#pragma unroll
        for (int i = 0; i < W; ++i) {
            const int t = s - (W - 1) + i;
            if (t < 0 || t >= p.T) continue;
            float dz[N];
            dz_row<T, W>(p, bh, t, c0, wv, bv, dz);
#pragma unroll
            for (int e = 0; e < N; ++e) g[e] = fmaf(wv[i][e], dz[e], g[e]);
        }
        if (p.dxs_out != nullptr && s >= p.T) {
            float go[N];
            load_vec(static_cast<const T*>(p.dxs_out) + ((size_t)bh * (W - 1) + (s - p.T)) * p.D + c0, go);
#pragma unroll
            for (int e = 0; e < N; ++e) g[e] += go[e];
        }
        store_vec(static_cast<T*>(p.dxs) + ((size_t)bh * (W - 1) + s) * p.D + c0, g);
    }
}

template <typename T, int W>
cudaError_t fwd_tw(const ConvParams& p, cudaStream_t s) {
    const int R = kThreads / (p.D / Vec<T>::N);
    const dim3 grid(p.B * p.H, (p.T + R * kRun - 1) / (R * kRun));
    if (p.T > 0) conv_fwd_kernel<T, W><<<grid, kThreads, 0, s>>>(p);
    if (p.xs_out && W > 1) {
        const size_t n = (size_t)p.B * p.H * (W - 1) * p.D;
        conv_state_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t bwd_tw(const ConvParams& p, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(p.dw, 0, (size_t)p.H * p.D * W * sizeof(float), s);
    if (e == cudaSuccess && p.dbias) e = cudaMemsetAsync(p.dbias, 0, (size_t)p.H * p.D * sizeof(float), s);
    if (e != cudaSuccess) return e;
    // tiles of `groups` R x kRun token groups: about four blocks per SM in all,
    // so each block sums the weight gradients over several groups before its
    // atomics
    const int R = kThreads / (p.D / Vec<T>::N);
    const int ngroups = (p.T + R * kRun - 1) / (R * kRun);
    const int want_tiles = std::max(1, (4 * sm_count() + p.B * p.H - 1) / (p.B * p.H));
    ConvParams q = p;
    q.conv_groups = std::max(1, (ngroups + want_tiles - 1) / want_tiles);
    const dim3 grid(p.B * p.H, (ngroups + q.conv_groups - 1) / q.conv_groups);
    if (p.T > 0) conv_bwd_kernel<T, W><<<grid, kThreads, 0, s>>>(q);
    if constexpr (W > 1) {
        if (p.dxs) {
            const size_t n = (size_t)p.B * p.H * (W - 1) * (p.D / Vec<T>::N);
            conv_state_grad_kernel<T, W><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
        }
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t fwd_t(const ConvParams& p, cudaStream_t s) {
    switch (p.W) {
        case 1: return fwd_tw<T, 1>(p, s);
        case 2: return fwd_tw<T, 2>(p, s);
        case 3: return fwd_tw<T, 3>(p, s);
        case 4: return fwd_tw<T, 4>(p, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t bwd_t(const ConvParams& p, cudaStream_t s) {
    switch (p.W) {
        case 1: return bwd_tw<T, 1>(p, s);
        case 2: return bwd_tw<T, 2>(p, s);
        case 3: return bwd_tw<T, 3>(p, s);
        case 4: return bwd_tw<T, 4>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_conv_fwd(const ConvParams& p, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    return p.bf16 ? fwd_t<__nv_bfloat16>(p, s) : fwd_t<float>(p, s);
}

cudaError_t launch_conv_bwd(const ConvParams& p, cudaStream_t s) {
    if (p.B * p.H == 0) {  // no tokens anywhere: the weight gradients are zero
        cudaError_t e = cudaMemsetAsync(p.dw, 0, (size_t)p.H * p.D * p.W * sizeof(float), s);
        if (e == cudaSuccess && p.dbias) e = cudaMemsetAsync(p.dbias, 0, (size_t)p.H * p.D * sizeof(float), s);
        return e;
    }
    return p.bf16 ? bwd_t<__nv_bfloat16>(p, s) : bwd_t<float>(p, s);
}

}  // namespace rdm
