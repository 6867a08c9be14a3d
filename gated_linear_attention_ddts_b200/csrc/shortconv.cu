// shortconv.cu -- the ShortConv of the Rodimus block: a causal depthwise
// convolution along the tokens (digest.lyk-ai.com summary of Rodimus*,
// "Method", third Rodimus bullet: a short convolution for local context next
// to the GLU; width, activation and carried state are this library's reading):
//
//   z[b,h,t,c] = bias[h,c] + sum_{i<W} w[h,c,i] x[b,h,t-i,c],   y = z or z*sigmoid(z)
//
// with x at t-i < 0 read from the carried-in state (the previous W-1 inputs).
//
// HBM-bound streaming through shared memory: persistent blocks take tiles of
// one (b, h) in turn (forward: 4096 elements, four blocks per SM; backward:
// 8192, two per SM).  The rows of a tile are contiguous in HBM; thread 0 keeps
// a ring of tiles in flight, each tile and its W-1 row halo arriving by one
// bulk copy (the backward: x and dy, halos on both sides), so the copy engine
// streams while the threads work out of shared memory on the tile before.
// Every thread takes a run of consecutive tokens of 4 channels and slides the
// staged rows through windows: the forward through a window of the last W
// inputs; the backward through one of inputs and one of dL/dz (z recomputed
// from the inputs when the SiLU is on), forming dx and the weight and bias
// gradients in a single sweep; those are reduced over the block (shuffles,
// then shared memory) before one float32 atomic per value and head.
#include <algorithm>

#include "conv_launch.h"
#include "launch.h"
#include "rdm_common.cuh"
#include "tc_ptx.cuh"

namespace rdm {
namespace {

using namespace tc;

constexpr int kThreads = 256;

// Four channels per thread (8 bytes of bf16, 16 of float32): small register
// footprints, so four blocks fit an SM and hide the shared-memory latencies.
template <typename T>
struct Vec {
    static constexpr int N = 4;
};

// inputs are read through the read-only path (x, dy and the states are never
// written by these kernels; the API requires outputs not to alias inputs), so
// the loads of a run can be issued ahead of its stores
__device__ __forceinline__ void load_vec(const float* p, float* f) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float* f) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void store_vec(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float* f) {
    uint2 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
    h[0] = __floats2bfloat162_rn(f[0], f[1]);
    h[1] = __floats2bfloat162_rn(f[2], f[3]);
    *reinterpret_cast<uint2*>(p) = u;
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

// SiLU(z) = z sigmoid(z) and d SiLU / dz = s (1 + z (1 - s)), s = sigmoid(z).
// float32 path: sigmoid through the fast reciprocal-based division
// (__fdividef: 2 ulp while the denominator 1 + e^-z is below 2^126, and 0
// beyond, where z e^z < 1e-36).  bf16 path, whose outputs carry 8 significant
// bits: sigmoid(z) = (1 + tanh(z/2)) / 2 with the single-instruction tanh
// (relative error about 2^-11), one MUFU operation per element instead of an
// exponential and a reciprocal.
template <typename T>
__device__ __forceinline__ float sigmoid_t(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
template <>
__device__ __forceinline__ float sigmoid_t<__nv_bfloat16>(float z) { return sigmoid_tanh(z); }
template <typename T>
__device__ __forceinline__ float silu_t(float z) { return z * sigmoid_t<T>(z); }
template <typename T>
__device__ __forceinline__ float silu_grad_t(float z) {
    const float s = sigmoid_t<T>(z);
    return s * (1.0f + z * (1.0f - s));
}

// 16 bytes of a staged row (shared memory) as floats
__device__ __forceinline__ void lds_vec(const float* p, float* f) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}
__device__ __forceinline__ void lds_vec(const __nv_bfloat16* p, float* f) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
}

// SiLU of the forward in three operations for bf16: with h = z/2,
// z sigmoid(z) = h (1 + tanh(h)) = fma(h, tanh(h), h).
template <typename T>
__device__ __forceinline__ float silu_fwd(float z) { return silu_t<T>(z); }
template <>
__device__ __forceinline__ float silu_fwd<__nv_bfloat16>(float z) {
    const float h = 0.5f * z;
    return fmaf(h, tanh_fast(h), h);
}

template <typename T>
__device__ __forceinline__ T zero_val() { return T(0.0f); }

constexpr int kConvStages = 4;     // tiles in flight per forward block
constexpr int kConvFwdRun = 4;     // consecutive tokens per forward thread
constexpr int kConvBwdStages = 2;  // per backward block (two blocks per SM fit)

// A tile: tokens [t0, t1) of sequence bh.
struct ConvTile {
    int bh, h, t0, t1;
};
__device__ __forceinline__ ConvTile conv_tile_of(const ConvParams& p, int g) {
    const int ntile = (p.T + p.tile - 1) / p.tile;
    ConvTile c;
    c.bh = g / ntile;
    c.h = c.bh % p.H;
    c.t0 = (g % ntile) * p.tile;
    c.t1 = min(c.t0 + p.tile, p.T);
    return c;
}

// The problems of one launch: problem i owns global tiles [tile0[i], tile0[i+1]).
struct ConvBatch {
    ConvParams p[kMaxConvBatch];
    int tile0[kMaxConvBatch + 1];
    int n;
    int stage;  // elements per ring stage: the largest of the problems'
};
__device__ __forceinline__ int conv_problem(const ConvBatch& m, int g) {
    int i = 0;
    while (i + 1 < m.n && g >= m.tile0[i + 1]) ++i;
    return i;
}

// Thread 0: bulk copy of the in-sequence rows [max(lo, 0), min(hi, T)) of
// sequence bh into dst, whose row 0 is token lo (the rows of one (b, h) are
// contiguous in HBM).  Returns the bytes it will deliver on `bar`.
template <typename T>
__device__ uint32_t copy_rows(const ConvParams& p, const T* seq, int bh, int lo, int hi, T* dst,
                              uint64_t* bar) {
    const int a = max(lo, 0), e = min(hi, p.T);
    if (a >= e) return 0u;
    const uint32_t bytes = (uint32_t)((size_t)(e - a) * p.D * sizeof(T));
    bulk_load(dst + (size_t)(a - lo) * p.D, seq + ((size_t)bh * p.T + a) * p.D, bytes, bar);
    return bytes;
}

// The rows of tokens lo .. -1 (lo < 0, the tile at the start of a sequence)
// from the carried-in state, zeros without one; all threads, then a barrier.
template <typename T, int W>
__device__ void fill_state_rows(const ConvParams& p, int bh, int lo, T* dst) {
    for (int i = threadIdx.x; i < -lo * p.D; i += kThreads) {
        const int s = W - 1 + lo + i / p.D;  // position in the carried-in state
        dst[i] = (p.xs && s >= 0) ? static_cast<const T*>(p.xs)[((size_t)bh * (W - 1) + s) * p.D + i % p.D]
                                  : zero_val<T>();
    }
    __syncthreads();
}

// Every thread waits (bounded) for phase `parity` of a stage; the block agrees
// (a wait that ran out sets the status word and the block leaves together).
__device__ __forceinline__ bool stage_ready(uint64_t* bar, uint32_t parity, const ConvParams& p) {
    const long long lim = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;
    const long long t0 = clock64();
    bool ok = true;
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > lim) {
            ok = false;
            break;
        }
    ok = __syncthreads_and(ok);
    if (!ok && threadIdx.x == 0) atomicOr(p.err, kErrTimeout);
    return ok;
}

// Before a block that gave up leaves: thread 0 waits (bounded) for the copies
// still in flight into its S stages (tiles k .. k + S - 1 that exist).
template <int S>
__device__ void drain_stages(uint64_t* full, int k, int g, int g1, const ConvParams& p) {
    if (threadIdx.x != 0) return;
    const long long lim = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;
    for (int j = 0; j < S && g + j < g1; ++j) {
        const int kk = k + j;
        const long long t0 = clock64();
        while (!mbar_try_wait(&full[kk % S], (kk / S) & 1) && clock64() - t0 <= lim) {
        }
    }
}

// Forward: persistent blocks (four per SM) take contiguous runs of tiles of
// `p.tile` tokens of one (b, h).  Thread 0 keeps kConvStages tiles in flight:
// each tile's rows and the W-1 rows before it arrive by one bulk copy into a
// ring stage; then thread (channel group cg, run of kConvFwdRun consecutive
// tokens) unpacks each staged row once, slides it through a window of the last
// W rows and stores 16 bytes of channels per token (8 for bf16).  Small tiles
// (4096 elements) give every block several, so that the first tiles' work
// overlaps the later tiles' copies.
template <typename T, int W, bool SILU>
__global__ void __launch_bounds__(kThreads, 4) conv_fwd_kernel(const __grid_constant__ ConvBatch m) {
    constexpr int N = Vec<T>::N, RUN = kConvFwdRun;
    extern __shared__ __align__(128) uint8_t conv_smem[];
    __shared__ uint64_t full[kConvStages];
    const int total = m.tile0[m.n];
    // a contiguous run of tiles per block (same sequence, mostly the same head);
    // the runs of the blocks differ by at most one tile
    const int g0 = (int)((long long)blockIdx.x * total / gridDim.x);
    const int g1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
    const size_t stage = (size_t)m.stage;
    T* ring = reinterpret_cast<T*>(conv_smem);
    const ConvParams& p0 = m.p[0];  // status word, wait bound and test hook (shared)
    auto issue = [&](int g, int s) {
        const int pi = conv_problem(m, g);
        const ConvParams& p = m.p[pi];
        const ConvTile c = conv_tile_of(p, g - m.tile0[pi]);
        mbar_expect_tx(&full[s], (uint32_t)((size_t)(c.t1 - max(c.t0 - (W - 1), 0)) * p.D * sizeof(T)));
        if (p.withhold) return;  // test hook: the stage never fills, its wait runs out
        copy_rows<T>(p, static_cast<const T*>(p.x), c.bh, c.t0 - (W - 1), c.t1, ring + s * stage, &full[s]);
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kConvStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kConvStages; ++s)
            if (g0 + s < g1) issue(g0 + s, s);
    }
    __syncthreads();
    float wv[W][N], bv[N];
    int cur_p = -1, cur_h = -1;
    int k = 0;
    for (int g = g0; g < g1; ++g, ++k) {
        const int s = k % kConvStages;
        const int pi = conv_problem(m, g);
        const ConvParams& p = m.p[pi];
        const ConvTile c = conv_tile_of(p, g - m.tile0[pi]);
        const int CG = p.D / N;
        const int cg = threadIdx.x % CG, run = threadIdx.x / CG, c0 = cg * N;
        const int lo = c.t0 - (W - 1);
        if (pi != cur_p || c.h != cur_h) {  // consecutive tiles mostly share the head
            cur_p = pi;
            cur_h = c.h;
#pragma unroll
            for (int e = 0; e < N; ++e) {
#pragma unroll
                for (int i = 0; i < W; ++i) wv[i][e] = __ldg(p.w + ((size_t)c.h * p.D + c0 + e) * W + i);
                bv[e] = p.bias ? __ldg(p.bias + (size_t)c.h * p.D + c0 + e) : 0.0f;
            }
        }
        if (!stage_ready(&full[s], (k / kConvStages) & 1, p0)) {
            drain_stages<kConvStages>(full, k, g, g1, p0);
            return;
        }
        T* xs = ring + s * stage;
        if (W > 1 && lo < 0) fill_state_rows<T, W>(p, c.bh, lo, xs);
        const int ta = c.t0 + run * RUN;
        if (ta < c.t1) {
            // staged row of token t at t - lo; my first window row is token ta - (W-1)
            const T* xr = xs + (size_t)(ta - (W - 1) - lo) * p.D + c0;
            T* yr = static_cast<T*>(p.y) + ((size_t)c.bh * p.T + ta) * p.D + c0;
            const int nrun = min(RUN, c.t1 - ta);
            float win[W][N];  // win[j] = x[t - (W-1) + j]
#pragma unroll
            for (int j = 0; j < W - 1; ++j) lds_vec(xr + (size_t)j * p.D, win[j]);
#pragma unroll
            for (int r = 0; r < RUN; ++r) {
                if (r >= nrun) break;
                lds_vec(xr + (size_t)(r + W - 1) * p.D, win[W - 1]);
                float z[N];
#pragma unroll
                for (int e = 0; e < N; ++e) {
                    float a = bv[e];
#pragma unroll
                    for (int i = 0; i < W; ++i) a = fmaf(wv[i][e], win[W - 1 - i][e], a);
                    z[e] = SILU ? silu_fwd<T>(a) : a;
                }
                store_vec(yr + (size_t)r * p.D, z);
#pragma unroll
                for (int j = 0; j < W - 1; ++j)
#pragma unroll
                    for (int e = 0; e < N; ++e) win[j][e] = win[j + 1][e];
            }
        }
        __syncthreads();  // stage s fully read: refill it with the tile kConvStages ahead
        if (threadIdx.x == 0 && g + kConvStages < g1) issue(g + kConvStages, s);
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
            dz[e] *= silu_grad_t<T>(a);
        }
    }
}

// Backward: persistent blocks (two per SM) with contiguous runs of tiles of
// 8192 elements, as in the forward.  A ring stage holds x of tokens
// [t0 - (W-1), t1 + W - 1) and dy of [t0, t1 + W - 1) (two bulk copies on one
// barrier).  Thread (channel group cg, run of kConvBwdRun consecutive tokens
// [ta, tb)) sweeps u over [ta, tb + W - 1) once: x[u] enters a window of the
// last W inputs, dL/dz[u] (dy through the SiLU, z recomputed from the window;
// zero past the end) enters a window of the last W of those, and
//   dx[u - (W-1)] = sum_i w_i dz[u - (W-1) + i]        (once the window is full)
//   dw_i += x[u - i] dz[u],  dbias += dz[u]             (u inside the run)
// so every staged row is read once per thread, plus the W-1 rows of halo on
// each side of its run.  The weight and bias partial sums are reduced over
// the block (shuffles, then shared memory) and added with one float32 atomic
// per value for each run of tiles of one head.
constexpr int kConvBwdRun = 8;
template <typename T, int W, bool SILU>
__global__ void __launch_bounds__(kThreads, 2) conv_bwd_kernel(const __grid_constant__ ConvBatch m) {
    constexpr int N = Vec<T>::N, RUN = kConvBwdRun;
    extern __shared__ __align__(128) uint8_t conv_smem[];
    __shared__ uint64_t full[kConvBwdStages];
    const int total = m.tile0[m.n];
    // contiguous runs of tiles that differ by at most one tile between blocks
    const int g0 = (int)((long long)blockIdx.x * total / gridDim.x);
    const int g1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
    const size_t stage = (size_t)m.stage;  // elements per ring stage
    T* ring = reinterpret_cast<T*>(conv_smem);
    float* s_red = reinterpret_cast<float*>(ring + kConvBwdStages * stage);  // [warps][D (W + 1)]
    const ConvParams& p0 = m.p[0];  // status word, wait bound and test hook (shared)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // a ring stage holds x of tokens [t0 - (W-1), t1 + W - 1), then dy of [t0, t1 + W - 1)
    auto issue = [&](int g, int s) {
        const int pi = conv_problem(m, g);
        const ConvParams& p = m.p[pi];
        const ConvTile c = conv_tile_of(p, g - m.tile0[pi]);
        const int lo = c.t0 - (W - 1), hi = c.t1 + W - 1;
        const size_t bx = (size_t)(min(hi, p.T) - max(lo, 0)) * p.D * sizeof(T);
        const size_t by = (size_t)(min(hi, p.T) - c.t0) * p.D * sizeof(T);
        mbar_expect_tx(&full[s], (uint32_t)(bx + by));
        if (p.withhold) return;  // test hook: the stage never fills, its wait runs out
        T* st = ring + s * stage;
        copy_rows<T>(p, static_cast<const T*>(p.x), c.bh, lo, hi, st, &full[s]);
        copy_rows<T>(p, static_cast<const T*>(p.dy), c.bh, c.t0, hi, st + (size_t)(p.tile + 2 * (W - 1)) * p.D,
                     &full[s]);
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kConvBwdStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        for (int s = 0; s < kConvBwdStages; ++s)
            if (g0 + s < g1) issue(g0 + s, s);
    }
    __syncthreads();
    float wv[W][N], bv[N], aw[W][N], ab[N];
    // weight and bias gradients summed over the block's tiles of head h of
    // problem pi: lanes holding the same channels (cg, cg + CG, ...) by shuffles,
    // one slot per warp in shared memory, a sum over the warps, one float32
    // atomic per value
    auto flush = [&](int pi, int h) {
        const ConvParams& p = m.p[pi];
        const int CG = p.D / N, cg = threadIdx.x % CG, DW1 = p.D * (W + 1);
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
            const int ch = gi * N + e;
            if (i < W) atomicAdd(p.dw + ((size_t)h * p.D + ch) * W + i, a);
            else if (p.dbias) atomicAdd(p.dbias + (size_t)h * p.D + ch, a);
        }
        __syncthreads();  // s_red read before it is written again
    };
    int cur_p = -1, cur_h = -1;
    int k = 0;
    for (int g = g0; g < g1; ++g, ++k) {
        const int s = k % kConvBwdStages;
        const int pi = conv_problem(m, g);
        const ConvParams& p = m.p[pi];
        const ConvTile c = conv_tile_of(p, g - m.tile0[pi]);
        const int CG = p.D / N;
        const int cg = threadIdx.x % CG, r0 = threadIdx.x / CG, c0 = cg * N;
        const int tout0 = p.T - (W - 1);  // first token copied into the carried-out state
        const int lo = c.t0 - (W - 1);
        if (pi != cur_p || c.h != cur_h) {  // block-uniform
            if (cur_p >= 0) flush(cur_p, cur_h);
            cur_p = pi;
            cur_h = c.h;
#pragma unroll
            for (int e = 0; e < N; ++e) {
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    wv[i][e] = __ldg(p.w + ((size_t)c.h * p.D + c0 + e) * W + i);
                    aw[i][e] = 0.0f;
                }
                bv[e] = p.bias ? __ldg(p.bias + (size_t)c.h * p.D + c0 + e) : 0.0f;
                ab[e] = 0.0f;
            }
        }
        if (!stage_ready(&full[s], (k / kConvBwdStages) & 1, p0)) {
            drain_stages<kConvBwdStages>(full, k, g, g1, p0);
            return;
        }
        T* xs = ring + s * stage;
        const T* dys = xs + (size_t)(p.tile + 2 * (W - 1)) * p.D;
        if (W > 1 && lo < 0) fill_state_rows<T, W>(p, c.bh, lo, xs);
        const int ta = c.t0 + r0 * RUN, tb = min(ta + RUN, c.t1);
        if (ta < c.t1) {
            // staged rows: x of token u at row u - lo, dy of token u at row u - t0;
            // rows at or past T are not staged and never enter a result
            T* dx = static_cast<T*>(p.dx) + (size_t)c.bh * p.T * p.D + c0;
            float xw[W][N];   // xw[j] = x[u - (W-1) + j] once x[u] is in
            float dzw[W][N];  // dzw[j] = dz[u - (W-1) + j] once dz[u] is in
#pragma unroll
            for (int j = 0; j < W - 1; ++j) lds_vec(xs + (size_t)(ta - (W - 1) + j - lo) * p.D + c0, xw[j]);
#pragma unroll
            for (int j = 0; j < W; ++j)
#pragma unroll
                for (int e = 0; e < N; ++e) dzw[j][e] = 0.0f;
#pragma unroll
            for (int k2 = 0; k2 < RUN + W - 1; ++k2) {
                const int u = ta + k2;
                if (u >= tb + W - 1) break;
                lds_vec(xs + (size_t)(u - lo) * p.D + c0, xw[W - 1]);
                float dz[N];
                if (u < p.T) {
                    lds_vec(dys + (size_t)(u - c.t0) * p.D + c0, dz);
                    if constexpr (SILU) {
#pragma unroll
                        for (int e = 0; e < N; ++e) {
                            float z = bv[e];
#pragma unroll
                            for (int i = 0; i < W; ++i) z = fmaf(wv[i][e], xw[W - 1 - i][e], z);
                            dz[e] *= silu_grad_t<T>(z);
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < N; ++e) dz[e] = 0.0f;
                }
                if (u < tb) {
#pragma unroll
                    for (int e = 0; e < N; ++e) {
#pragma unroll
                        for (int i = 0; i < W; ++i) aw[i][e] = fmaf(xw[W - 1 - i][e], dz[e], aw[i][e]);
                        ab[e] += dz[e];
                    }
                }
#pragma unroll
                for (int j = 0; j < W - 1; ++j)
#pragma unroll
                    for (int e = 0; e < N; ++e) dzw[j][e] = dzw[j + 1][e];
#pragma unroll
                for (int e = 0; e < N; ++e) dzw[W - 1][e] = dz[e];
                if (k2 >= W - 1) {
                    const int t = u - (W - 1);  // in [ta, tb)
                    float gx[N];
#pragma unroll
                    for (int e = 0; e < N; ++e) {
                        float a = 0.0f;
#pragma unroll
                        for (int i = 0; i < W; ++i) a = fmaf(wv[i][e], dzw[i][e], a);
                        gx[e] = a;
                    }
                    if (p.dxs_out != nullptr && t >= tout0) {
                        float go[N];
                        load_vec(static_cast<const T*>(p.dxs_out) + ((size_t)c.bh * (W - 1) + (t - tout0)) * p.D + c0, go);
#pragma unroll
                        for (int e = 0; e < N; ++e) gx[e] += go[e];
                    }
                    store_vec(dx + (size_t)t * p.D, gx);
                }
#pragma unroll
                for (int j = 0; j < W - 1; ++j)
#pragma unroll
                    for (int e = 0; e < N; ++e) xw[j][e] = xw[j + 1][e];
            }
        }
        __syncthreads();  // stage s fully read: refill it
        if (threadIdx.x == 0 && g + kConvBwdStages < g1) issue(g + kConvBwdStages, s);
    }
    if (cur_p >= 0) flush(cur_p, cur_h);
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

// Tokens per tile: a run of kConvFwdRun (forward: 4096 elements, 64 tokens at
// D = 64) or kConvBwdRun (backward: 8192 elements) tokens for every thread.
int conv_tile(const ConvParams& p) { return kConvFwdRun * kThreads / (p.D / Vec<float>::N); }
int conv_tile_bwd(const ConvParams& p) { return kConvBwdRun * kThreads / (p.D / Vec<float>::N); }

// The batch of a launch: tiles of each problem, their index space, the largest
// ring stage.  Returns the number of tiles.
template <int W>
int make_batch(ConvBatch& m, const ConvParams* ps, int n, bool bwd, size_t elem) {
    m.n = n;
    int total = 0;
    size_t stage = 0;
    for (int i = 0; i < n; ++i) {
        ConvParams p = ps[i];
        p.tile = bwd ? conv_tile_bwd(p) : conv_tile(p);
        m.p[i] = p;
        m.tile0[i] = total;
        if (p.T > 0) total += p.B * p.H * ((p.T + p.tile - 1) / p.tile);
        const size_t rows = bwd ? (size_t)2 * p.tile + 3 * (W - 1) : (size_t)p.tile + W - 1;
        stage = std::max(stage, rows * p.D);
    }
    m.tile0[n] = total;
    // keep every stage 128-byte aligned (bulk copies need 16)
    const size_t q = 128 / elem;
    m.stage = (int)((stage + q - 1) / q * q);
    return total;
}

// Persistent grid: `per_sm` blocks per SM, or fewer when there are fewer tiles.
unsigned conv_grid(int tiles, int per_sm) {
    const long long cap = (long long)per_sm * sm_count();
    return (unsigned)(tiles < cap ? tiles : cap);
}

template <typename T, int W>
cudaError_t fwd_tw(const ConvParams* ps, int n, cudaStream_t s) {
    ConvBatch m;
    const int tiles = make_batch<W>(m, ps, n, false, sizeof(T));
    if (tiles > 0) {
        const size_t smem = (size_t)kConvStages * m.stage * sizeof(T);
        auto kern = ps[0].silu ? conv_fwd_kernel<T, W, true> : conv_fwd_kernel<T, W, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<conv_grid(tiles, 4), kThreads, smem, s>>>(m);
    }
    for (int i = 0; i < n; ++i) {
        const ConvParams& p = ps[i];
        if (p.xs_out && W > 1) {
            const size_t ne = (size_t)p.B * p.H * (W - 1) * p.D;
            conv_state_kernel<T><<<(unsigned)((ne + 255) / 256), 256, 0, s>>>(p);
        }
    }
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t bwd_tw(const ConvParams* ps, int n, cudaStream_t s) {
    for (int i = 0; i < n; ++i) {
        const ConvParams& p = ps[i];
        cudaError_t e = cudaMemsetAsync(p.dw, 0, (size_t)p.H * p.D * W * sizeof(float), s);
        if (e == cudaSuccess && p.dbias) e = cudaMemsetAsync(p.dbias, 0, (size_t)p.H * p.D * sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    ConvBatch m;
    const int tiles = make_batch<W>(m, ps, n, true, sizeof(T));
    if (tiles > 0) {
        int dmax = 0;
        for (int i = 0; i < n; ++i) dmax = std::max(dmax, ps[i].D);
        const size_t smem = (size_t)kConvBwdStages * m.stage * sizeof(T) +
                            (size_t)(kThreads / 32) * dmax * (W + 1) * 4;
        auto kern = ps[0].silu ? conv_bwd_kernel<T, W, true> : conv_bwd_kernel<T, W, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<conv_grid(tiles, 2), kThreads, smem, s>>>(m);
    }
    if constexpr (W > 1) {
        for (int i = 0; i < n; ++i) {
            const ConvParams& p = ps[i];
            if (p.dxs && p.B * p.H > 0) {
                const size_t ne = (size_t)p.B * p.H * (W - 1) * (p.D / Vec<T>::N);
                conv_state_grad_kernel<T, W><<<(unsigned)((ne + 255) / 256), 256, 0, s>>>(p);
            }
        }
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t fwd_t(const ConvParams* ps, int n, cudaStream_t s) {
    switch (ps[0].W) {
        case 1: return fwd_tw<T, 1>(ps, n, s);
        case 2: return fwd_tw<T, 2>(ps, n, s);
        case 3: return fwd_tw<T, 3>(ps, n, s);
        case 4: return fwd_tw<T, 4>(ps, n, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t bwd_t(const ConvParams* ps, int n, cudaStream_t s) {
    switch (ps[0].W) {
        case 1: return bwd_tw<T, 1>(ps, n, s);
        case 2: return bwd_tw<T, 2>(ps, n, s);
        case 3: return bwd_tw<T, 3>(ps, n, s);
        case 4: return bwd_tw<T, 4>(ps, n, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_conv_fwd_many(const ConvParams* ps, int n, cudaStream_t s) {
    if (n < 1 || n > kMaxConvBatch) return cudaErrorInvalidValue;
    return ps[0].bf16 ? fwd_t<__nv_bfloat16>(ps, n, s) : fwd_t<float>(ps, n, s);
}

cudaError_t launch_conv_bwd_many(const ConvParams* ps, int n, cudaStream_t s) {
    if (n < 1 || n > kMaxConvBatch) return cudaErrorInvalidValue;
    // a problem without tokens (B*H == 0 or T == 0) still gets its weight
    // gradients zeroed by the memsets
    return ps[0].bf16 ? bwd_t<__nv_bfloat16>(ps, n, s) : bwd_t<float>(ps, n, s);
}

cudaError_t launch_conv_fwd(const ConvParams& p, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    return launch_conv_fwd_many(&p, 1, s);
}

cudaError_t launch_conv_bwd(const ConvParams& p, cudaStream_t s) { return launch_conv_bwd_many(&p, 1, s); }

}  // namespace rdm
