// shortconv.cu -- the ShortConv of the Rodimus block: a causal depthwise
// convolution along the tokens (digest.lyk-ai.com summary of Rodimus*,
// "Method", third Rodimus bullet: a short convolution for local context next
// to the GLU; width, activation and carried state are this library's reading):
//
//   z[b,h,t,c] = bias[h,c] + sum_{i<W} w[h,c,i] x[b,h,t-i,c],   y = z or z*sigmoid(z)
//
// with x at t-i < 0 read from the carried-in state (the previous W-1 inputs).
//
// HBM-bound streaming through shared memory: a block takes a tile of tokens of
// one (b, h) (8192 elements, 128 tokens at D = 64), whose rows are contiguous
// in HBM, and has the bulk copy engine bring the tile and its W-1 row halo
// into shared memory in one transfer (the backward: x and dy, with the halo on
// both sides); the threads then work out of shared memory, 16 bytes of
// channels of one token at a time, and store whole rows.  The backward first
// writes dL/dz of the tile to shared memory (z recomputed from the staged x
// when the SiLU is on), then forms dx and the weight and bias gradients, which
// are reduced over the block (shuffles, then shared memory) before one float32
// atomic per value and block.
#include <algorithm>

#include "launch.h"
#include "rdm_common.cuh"
#include "tc_ptx.cuh"

namespace rdm {
namespace {

using namespace tc;

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

// 16 bytes of a staged row (shared memory) as floats
__device__ __forceinline__ void lds_vec(const float* p, float* f) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}
__device__ __forceinline__ void lds_vec(const __nv_bfloat16* p, float* f) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

template <typename T>
__device__ __forceinline__ T zero_val() { return T(0.0f); }

// Stage the rows of tokens [lo, hi) of sequence bh (rows of D elements) into
// dst: the in-sequence rows [max(lo, 0), min(hi, T)) are handed to the bulk
// copy engine by thread 0 (the rows of one (b, h) are contiguous in HBM);
// tokens before the sequence come from the carried-in state (zeros without
// one, or when `state` is null), tokens past its end are zeros.  Returns the
// bytes the bulk copy will deliver on `bar`.
template <typename T, int W>
__device__ uint32_t stage_rows(const ConvParams& p, const T* seq, const T* state, int bh, int lo,
                               int hi, T* dst, uint64_t* bar) {
    const int a = max(lo, 0), e = min(hi, p.T);
    const uint32_t bytes = a < e ? (uint32_t)((size_t)(e - a) * p.D * sizeof(T)) : 0u;
    if (threadIdx.x == 0 && bytes)
        bulk_load(dst + (size_t)(a - lo) * p.D, seq + ((size_t)bh * p.T + a) * p.D, bytes, bar);
    for (int i = threadIdx.x; i < (a - lo) * p.D; i += kThreads) {
        const int s = W - 1 + lo + i / p.D;  // position in the carried-in state
        dst[i] = (state && s >= 0) ? state[((size_t)bh * (W - 1) + s) * p.D + i % p.D] : zero_val<T>();
    }
    for (int i = (e - lo) * p.D + threadIdx.x; i < (hi - lo) * p.D; i += kThreads)
        dst[i] = zero_val<T>();
    return bytes;
}

// Every thread waits (bounded) for the staged rows.  A wait that runs out sets
// the status word; the thread then waits once more, also bounded, so that no
// copy lands after the block has left, and the block skips its work.
__device__ __forceinline__ bool staged(uint64_t* bar, const ConvParams& p) {
    const long long lim = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, 0))
        if (clock64() - t0 > lim) {
            atomicOr(p.err, kErrTimeout);
            t0 = clock64();
            while (!mbar_try_wait(bar, 0) && clock64() - t0 <= lim) {
            }
            return false;
        }
    return true;
}

// Forward: one block per tile of `p.tile` tokens of one (b, h).  The tile's
// inputs and the W-1 rows before it are staged in shared memory by one bulk
// copy; then thread (channel group cg, token lane r) produces 16 bytes of
// channels for tokens t0 + r, t0 + r + R, ... (a warp stores whole rows).
template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv_fwd_kernel(const ConvParams p) {
    constexpr int N = Vec<T>::N;
    extern __shared__ __align__(128) uint8_t conv_smem[];
    __shared__ uint64_t bar;
    T* xs = reinterpret_cast<T*>(conv_smem);  // rows of tokens [t0 - (W-1), t1)
    const int CG = p.D / N, R = kThreads / CG;
    const int ntile = (p.T + p.tile - 1) / p.tile;
    const int bh = blockIdx.x / ntile, h = bh % p.H;
    const int t0 = (blockIdx.x % ntile) * p.tile, t1 = min(t0 + p.tile, p.T);
    const int lo = t0 - (W - 1);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t bytes = stage_rows<T, W>(p, static_cast<const T*>(p.x), static_cast<const T*>(p.xs),
                                            bh, lo, t1, xs, &bar);
    if (threadIdx.x == 0) mbar_expect_tx(&bar, bytes);
    const int cg = threadIdx.x % CG, r0 = threadIdx.x / CG, c0 = cg * N;
    float wv[W][N], bv[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i < W; ++i) wv[i][e] = __ldg(p.w + ((size_t)h * p.D + c0 + e) * W + i);
        bv[e] = p.bias ? __ldg(p.bias + (size_t)h * p.D + c0 + e) : 0.0f;
    }
    __syncthreads();  // the rows the threads filled
    if (!__syncthreads_and(staged(&bar, p))) return;  // the block leaves together
    T* y = static_cast<T*>(p.y) + (size_t)bh * p.T * p.D + c0;
    for (int t = t0 + r0; t < t1; t += R) {
        float z[N];
#pragma unroll
        for (int e = 0; e < N; ++e) z[e] = bv[e];
#pragma unroll
        for (int i = 0; i < W; ++i) {
            float xv[N];
            lds_vec(xs + (size_t)(t - i - lo) * p.D + c0, xv);
#pragma unroll
            for (int e = 0; e < N; ++e) z[e] = fmaf(wv[i][e], xv[e], z[e]);
        }
        if (p.silu) {
#pragma unroll
            for (int e = 0; e < N; ++e) z[e] = silu_f(z[e]);
        }
        store_vec(y + (size_t)t * p.D, z);
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

// Backward: one block per tile of `p.tile` tokens of one (b, h).  Staged: x of
// tokens [t0 - (W-1), t1 + W - 1) and dy of [t0, t1 + W - 1) (bulk copies, as
// in the forward).  Phase 1 writes dL/dz of tokens [t0, t1 + W - 1) (zero past
// the end) to shared memory as float32; phase 2 gives dx[t] = sum_i w_i dz[t+i]
// (plus the carried-out state's gradient where it copies x[t]) and accumulates
// the weight and bias gradients, which are summed over the block and added
// with one float32 atomic per value.
template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv_bwd_kernel(const ConvParams p) {
    constexpr int N = Vec<T>::N;
    extern __shared__ __align__(128) uint8_t conv_smem[];
    __shared__ uint64_t bar;
    const int TT = p.tile;
    const int ntile = (p.T + TT - 1) / TT;
    const int bh = blockIdx.x / ntile, h = bh % p.H;
    const int t0 = (blockIdx.x % ntile) * TT, t1 = min(t0 + TT, p.T);
    const int lo = t0 - (W - 1), hi = t1 + W - 1;   // x rows [lo, hi)
    const int nz = hi - t0;                          // dz and dy rows [t0, hi)
    T* xs = reinterpret_cast<T*>(conv_smem);
    T* dys = xs + (size_t)(TT + 2 * (W - 1)) * p.D;
    float* dzs = reinterpret_cast<float*>(dys + (size_t)(TT + W - 1) * p.D);
    float* s_red = dzs + (size_t)(TT + W - 1) * p.D;   // [warps][D (W + 1)]
    const int CG = p.D / N, R = kThreads / CG;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t bytes = stage_rows<T, W>(p, static_cast<const T*>(p.x), static_cast<const T*>(p.xs), bh,
                                      lo, hi, xs, &bar);
    bytes += stage_rows<T, W>(p, static_cast<const T*>(p.dy), nullptr, bh, t0, hi, dys, &bar);
    if (threadIdx.x == 0) mbar_expect_tx(&bar, bytes);
    const int cg = threadIdx.x % CG, r0 = threadIdx.x / CG, c0 = cg * N;
    float wv[W][N], bv[N], aw[W][N], ab[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i < W; ++i) {
            wv[i][e] = __ldg(p.w + ((size_t)h * p.D + c0 + e) * W + i);
            aw[i][e] = 0.0f;
        }
        bv[e] = p.bias ? __ldg(p.bias + (size_t)h * p.D + c0 + e) : 0.0f;
        ab[e] = 0.0f;
    }
    __syncthreads();  // the rows the threads filled
    if (!__syncthreads_and(staged(&bar, p))) return;  // the block leaves together
    // phase 1: dz = dy, through the SiLU when on (z recomputed from the staged x)
    for (int u = r0; u < nz; u += R) {
        const int t = t0 + u;
        float dz[N];
        if (t < p.T) {
            lds_vec(dys + (size_t)u * p.D + c0, dz);
            if (p.silu) {
                float z[N];
#pragma unroll
                for (int e = 0; e < N; ++e) z[e] = bv[e];
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    float xv[N];
                    lds_vec(xs + (size_t)(t - i - lo) * p.D + c0, xv);
#pragma unroll
                    for (int e = 0; e < N; ++e) z[e] = fmaf(wv[i][e], xv[e], z[e]);
                }
#pragma unroll
                for (int e = 0; e < N; ++e) dz[e] *= silu_grad(z[e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < N; ++e) dz[e] = 0.0f;
        }
        float* row = dzs + (size_t)u * p.D + c0;
#pragma unroll
        for (int e = 0; e < N; e += 4) *reinterpret_cast<float4*>(row + e) = make_float4(dz[e], dz[e + 1], dz[e + 2], dz[e + 3]);
    }
    __syncthreads();
    // phase 2
    T* dx = static_cast<T*>(p.dx) + (size_t)bh * p.T * p.D + c0;
    const int tout0 = p.T - (W - 1);  // first token copied into the carried-out state
    for (int t = t0 + r0; t < t1; t += R) {
        const int u = t - t0;
        float dzr[W][N];
#pragma unroll
        for (int i = 0; i < W; ++i)
#pragma unroll
            for (int e = 0; e < N; e += 4) {
                const float4 f = *reinterpret_cast<const float4*>(dzs + (size_t)(u + i) * p.D + c0 + e);
                dzr[i][e] = f.x; dzr[i][e + 1] = f.y; dzr[i][e + 2] = f.z; dzr[i][e + 3] = f.w;
            }
        float g[N];
#pragma unroll
        for (int e = 0; e < N; ++e) {
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < W; ++i) a = fmaf(wv[i][e], dzr[i][e], a);
            g[e] = a;
            ab[e] += dzr[0][e];
        }
#pragma unroll
        for (int i = 0; i < W; ++i) {
            float xv[N];
            lds_vec(xs + (size_t)(t - i - lo) * p.D + c0, xv);
#pragma unroll
            for (int e = 0; e < N; ++e) aw[i][e] = fmaf(dzr[0][e], xv[e], aw[i][e]);
        }
        if (p.dxs_out != nullptr && t >= tout0) {
            float go[N];
            load_vec(static_cast<const T*>(p.dxs_out) + ((size_t)bh * (W - 1) + (t - tout0)) * p.D + c0, go);
#pragma unroll
            for (int e = 0; e < N; ++e) g[e] += go[e];
        }
        store_vec(dx + (size_t)t * p.D, g);
    }
    // weight and bias gradients: the lanes of a warp that hold the same channels
    // (lanes cg, cg + CG, ...) by shuffles, one slot per warp in shared memory,
    // a sum over the warps, then one float32 atomic per value and block
    const int DW1 = p.D * (W + 1);
#pragma unroll
    for (int e = 0; e < N; ++e) {
#pragma unroll
        for (int i = 0; i <= W; ++i) {
            float x = i < W ? aw[i][e] : ab[e];
            for (int off = CG; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (lane < CG) s_red[warp * DW1 + (cg * (W + 1) + i) * N + e] = x;
        }
    }
    __syncthreads();
    // CG divides 32 (D / N <= 32), so every warp holds every channel group
    for (int idx = threadIdx.x; idx < DW1; idx += kThreads) {
        const int e = idx % N, i = (idx / N) % (W + 1), gi = idx / (N * (W + 1));
        float a = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < kThreads / 32; ++w2) a += s_red[w2 * DW1 + idx];
        const int c = gi * N + e;
        if (i < W) atomicAdd(p.dw + ((size_t)h * p.D + c) * W + i, a);
        else if (p.dbias) atomicAdd(p.dbias + (size_t)h * p.D + c, a);
    }
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

// Tokens per block: tiles of 8192 elements (128 tokens at D = 64), at least W.
int conv_tile(const ConvParams& p) { return std::max(8192 / p.D, 8); }

template <typename T, int W>
size_t fwd_smem(const ConvParams& p) {
    return (size_t)(p.tile + W - 1) * p.D * sizeof(T);
}

template <typename T, int W>
size_t bwd_smem(const ConvParams& p) {
    return (size_t)(p.tile + 2 * (W - 1)) * p.D * sizeof(T) + (size_t)(p.tile + W - 1) * p.D * sizeof(T) +
           (size_t)(p.tile + W - 1) * p.D * 4 + (size_t)(kThreads / 32) * p.D * (W + 1) * 4;
}

template <typename T, int W>
cudaError_t fwd_tw(const ConvParams& p0, cudaStream_t s) {
    ConvParams p = p0;
    p.tile = conv_tile(p);
    if (p.T > 0) {
        const size_t smem = fwd_smem<T, W>(p);
        auto kern = conv_fwd_kernel<T, W>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const unsigned grid = (unsigned)((size_t)p.B * p.H * ((p.T + p.tile - 1) / p.tile));
        kern<<<grid, kThreads, smem, s>>>(p);
    }
    if (p.xs_out && W > 1) {
        const size_t n = (size_t)p.B * p.H * (W - 1) * p.D;
        conv_state_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t bwd_tw(const ConvParams& p0, cudaStream_t s) {
    ConvParams p = p0;
    p.tile = conv_tile(p);
    cudaError_t e = cudaMemsetAsync(p.dw, 0, (size_t)p.H * p.D * W * sizeof(float), s);
    if (e == cudaSuccess && p.dbias) e = cudaMemsetAsync(p.dbias, 0, (size_t)p.H * p.D * sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (p.T > 0) {
        const size_t smem = bwd_smem<T, W>(p);
        auto kern = conv_bwd_kernel<T, W>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const unsigned grid = (unsigned)((size_t)p.B * p.H * ((p.T + p.tile - 1) / p.tile));
        kern<<<grid, kThreads, smem, s>>>(p);
    }
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
