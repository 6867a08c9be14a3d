// simt.cu -- exact token-serial DDTS recurrence on CUDA cores (float32
// arithmetic, float32 or bf16 storage).  This is the float32 path and the
// path for shapes the tensor-core kernels do not take.
//
// Forward (per (b,h), one block; thread j owns column j of the state):
//     S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t k_t)(beta_hat_t v_t)^T,  o_t = S_t^T q_t
// (Rodimus*, digest.lyk-ai.com summary "Method" for the gates; diagonal decay
// along d_k per the paperhub.cn rebuttal "Efficient Parallelization" bullet.)
//
// Backward, exact reverse mode organised in two sweeps per (b,h), thread i
// owning row i of the state or of its gradient:
//   sweep F (forward in t):  S_t, dq_t = S_t dO_t, and q_t*dq_t kept in scratch;
//   sweep R (reverse in t):  dS_t = q_t dO_t^T + diag(alpha_{t+1}) dS_{t+1},
//                            dkhat_t = dS_t vhat_t, dvhat_t = dS_t^T khat_t.
// The decay gradient uses d(log alpha_t) = sum_{u>=t} dG_u with
//   dG_u = q_u*dq_u - khat_u*dkhat_u  (+ rowsum(dS_T o S_T) at u = T),
// which follows from S_t = sum_s diag(exp(G_t - G_s)) khat_s vhat_s^T + diag(exp(G_t)) S_0
// with G_t the running sum of log alpha.
#include "launch.h"
#include "rdm_common.cuh"

namespace rdm {
namespace {

constexpr int kTile = 16;  // tokens staged in shared memory at a time

// ------------------------------------------------------------------ forward
template <typename T, int DK>
__global__ void __launch_bounds__(128) simt_fwd_kernel(SeqParams p) {
    const int bh = blockIdx.x;
    const int j = threadIdx.x;  // column of the state owned by this thread
    const int T_ = p.T, dv = p.dv;
    const int NC = (T_ + p.chunk - 1) / p.chunk;
    __shared__ float s_al[kTile][DK], s_kh[kTile][DK], s_q[kTile][DK];

    const T* q = static_cast<const T*>(p.q) + (size_t)bh * T_ * DK;
    const T* k = static_cast<const T*>(p.k) + (size_t)bh * T_ * DK;
    const T* g = static_cast<const T*>(p.g) + (size_t)bh * T_ * DK;
    const T* tau = static_cast<const T*>(p.tau) + (size_t)bh * T_ * DK;
    const T* v = static_cast<const T*>(p.v) + (size_t)bh * T_ * dv;
    const T* beta = static_cast<const T*>(p.beta) + (size_t)bh * T_ * dv;
    T* o = static_cast<T*>(p.o) + (size_t)bh * T_ * dv;

    float s[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i)
        s[i] = p.S0 ? p.S0[((size_t)bh * DK + i) * dv + j] : 0.0f;

    for (int t0 = 0; t0 < T_; t0 += kTile) {
        const int nt = min(kTile, T_ - t0);
        for (int idx = threadIdx.x; idx < nt * DK; idx += blockDim.x) {
            const int tt = idx / DK, i = idx % DK;
            const size_t off = (size_t)(t0 + tt) * DK + i;
            float gg = ldf(g + off), ta = ldf(tau + off);
            if (p.preact) {
                gg = softplus_acc(gg);
                ta = sigmoid_acc(ta);
            }
            s_al[tt][i] = alpha(gg, ta);
            s_kh[tt][i] = alpha_hat(gg, ta) * ldf(k + off);
            s_q[tt][i] = ldf(q + off);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const int t = t0 + tt;
            if (p.saved && t % p.chunk == 0) {
                float* dst = p.saved + (((size_t)bh * NC + t / p.chunk) * DK) * dv + j;
#pragma unroll
                for (int i = 0; i < DK; ++i) dst[(size_t)i * dv] = s[i];
            }
            const float bb = ldf(beta + (size_t)t * dv + j);
            const float vt = ldf(v + (size_t)t * dv + j);
            const float vh = (p.preact ? sigmoid_acc(bb) : bb) * vt;
            // feedthrough o_t += d (.) v_t
            float acc = p.dfeed ? p.dfeed[(size_t)(bh % p.H) * dv + j] * vt : 0.0f;
#pragma unroll
            for (int i = 0; i < DK; ++i) {
                s[i] = fmaf(s_al[tt][i], s[i], s_kh[tt][i] * vh);
                acc = fmaf(s[i], s_q[tt][i], acc);
            }
            stf(o + (size_t)t * dv + j, acc);
        }
        __syncthreads();
    }
    if (p.ST) {
#pragma unroll
        for (int i = 0; i < DK; ++i) p.ST[((size_t)bh * DK + i) * dv + j] = s[i];
    }
}

// ------------------------------------------------ backward, forward sweep F
template <typename T, int DV>
__global__ void __launch_bounds__(128) simt_bwd_fsweep(BwdParams p, float* qdq, float* fin,
                                                       const int* only) {
    const int bh = blockIdx.x;
    if (only && only[bh] == 0) return;  // head already handled by the tensor-core path
    const int T_ = p.T, dk = p.dk;
    const bool act = (int)threadIdx.x < dk;  // block padded to whole warps
    const int i = act ? threadIdx.x : 0;      // row of the state owned by this thread
    __shared__ float s_vh[kTile][DV], s_do[kTile][DV];

    const T* q = static_cast<const T*>(p.q) + (size_t)bh * T_ * dk;
    const T* k = static_cast<const T*>(p.k) + (size_t)bh * T_ * dk;
    const T* g = static_cast<const T*>(p.g) + (size_t)bh * T_ * dk;
    const T* tau = static_cast<const T*>(p.tau) + (size_t)bh * T_ * dk;
    const T* v = static_cast<const T*>(p.v) + (size_t)bh * T_ * DV;
    const T* beta = static_cast<const T*>(p.beta) + (size_t)bh * T_ * DV;
    const T* dO = static_cast<const T*>(p.dO) + (size_t)bh * T_ * DV;
    T* dq = static_cast<T*>(p.dq) + (size_t)bh * T_ * dk;
    float* qdq_bh = qdq + (size_t)bh * T_ * dk;

    float s[DV];
#pragma unroll
    for (int j = 0; j < DV; ++j) s[j] = p.S0 ? p.S0[((size_t)bh * dk + i) * DV + j] : 0.0f;

    for (int t0 = 0; t0 < T_; t0 += kTile) {
        const int nt = min(kTile, T_ - t0);
        for (int idx = threadIdx.x; idx < nt * DV; idx += blockDim.x) {
            const int tt = idx / DV, j = idx % DV;
            const size_t off = (size_t)(t0 + tt) * DV + j;
            const float bb = ldf(beta + off);
            s_vh[tt][j] = (p.preact ? sigmoid_acc(bb) : bb) * ldf(v + off);
            s_do[tt][j] = ldf(dO + off);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const size_t off = (size_t)(t0 + tt) * dk + i;
            float gg = ldf(g + off), ta = ldf(tau + off);
            if (p.preact) {
                gg = softplus_acc(gg);
                ta = sigmoid_acc(ta);
            }
            const float al = alpha(gg, ta), kh = alpha_hat(gg, ta) * ldf(k + off);
            float acc = 0.0f;
#pragma unroll
            for (int j = 0; j < DV; ++j) {
                s[j] = fmaf(al, s[j], kh * s_vh[tt][j]);
                acc = fmaf(s[j], s_do[tt][j], acc);
            }
            if (act) {
                stf(dq + off, acc);
                qdq_bh[off] = ldf(q + off) * acc;
            }
        }
        __syncthreads();
    }
    float f = 0.0f;
    if (p.dST) {
#pragma unroll
        for (int j = 0; j < DV; ++j) f = fmaf(p.dST[((size_t)bh * dk + i) * DV + j], s[j], f);
    }
    if (act) fin[(size_t)bh * dk + i] = f;
}

// ------------------------------------------------ backward, reverse sweep R
template <typename T, int DV>
__global__ void __launch_bounds__(128) simt_bwd_rsweep(BwdParams p, const float* qdq,
                                                       const float* fin, const int* only) {
    const int bh = blockIdx.x;
    if (only && only[bh] == 0) return;
    const int T_ = p.T, dk = p.dk;
    // the block is padded to whole warps; rows past d_k carry zeros
    const bool act = (int)threadIdx.x < dk;
    const int i = act ? threadIdx.x : 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x / 32;
    __shared__ float s_vh[kTile][DV], s_do[kTile][DV], s_red[4][DV];

    const T* q = static_cast<const T*>(p.q) + (size_t)bh * T_ * dk;
    const T* k = static_cast<const T*>(p.k) + (size_t)bh * T_ * dk;
    const T* g = static_cast<const T*>(p.g) + (size_t)bh * T_ * dk;
    const T* tau = static_cast<const T*>(p.tau) + (size_t)bh * T_ * dk;
    const T* v = static_cast<const T*>(p.v) + (size_t)bh * T_ * DV;
    const T* beta = static_cast<const T*>(p.beta) + (size_t)bh * T_ * DV;
    const T* dO = static_cast<const T*>(p.dO) + (size_t)bh * T_ * DV;
    T* dk_ = static_cast<T*>(p.dk_) + (size_t)bh * T_ * dk;
    T* dg = static_cast<T*>(p.dg) + (size_t)bh * T_ * dk;
    T* dtau = static_cast<T*>(p.dtau) + (size_t)bh * T_ * dk;
    T* dv_ = static_cast<T*>(p.dv_) + (size_t)bh * T_ * DV;
    T* dbeta = static_cast<T*>(p.dbeta) + (size_t)bh * T_ * DV;
    const float* qdq_bh = qdq + (size_t)bh * T_ * dk;

    float ds[DV];
#pragma unroll
    for (int j = 0; j < DV; ++j)
        ds[j] = (act && p.dST) ? p.dST[((size_t)bh * dk + i) * DV + j] : 0.0f;
    float a_next = 1.0f;                  // alpha_{t+1,i}
    float da = fin[(size_t)bh * dk + i];  // running sum of dG over u >= t

    for (int t1 = T_; t1 > 0; t1 -= kTile) {
        const int t0 = max(0, t1 - kTile), nt = t1 - t0;
        for (int idx = threadIdx.x; idx < nt * DV; idx += blockDim.x) {
            const int tt = idx / DV, j = idx % DV;
            const size_t off = (size_t)(t0 + tt) * DV + j;
            const float bb = ldf(beta + off);
            s_vh[tt][j] = (p.preact ? sigmoid_acc(bb) : bb) * ldf(v + off);
            s_do[tt][j] = ldf(dO + off);
        }
        __syncthreads();
        for (int tt = nt - 1; tt >= 0; --tt) {
            const size_t off = (size_t)(t0 + tt) * dk + i;
            const float g_in = ldf(g + off), t_in = ldf(tau + off), kk = ldf(k + off);
            const float gg = p.preact ? softplus_acc(g_in) : g_in;
            const float ta = p.preact ? sigmoid_acc(t_in) : t_in;
            // chain factors to the pre-activations: softplus' = sigmoid, sigmoid' = s (1 - s)
            const float cg = p.preact ? sigmoid_acc(g_in) : 1.0f;
            const float ct = p.preact ? ta * (1.0f - ta) : 1.0f;
            const float qi = act ? ldf(q + off) : 0.0f;
            const float al = alpha(gg, ta), ah = alpha_hat(gg, ta);
            const float kh = act ? ah * kk : 0.0f;
            float dkh = 0.0f;
#pragma unroll
            for (int j = 0; j < DV; ++j) {
                ds[j] = fmaf(a_next, ds[j], qi * s_do[tt][j]);
                dkh = fmaf(ds[j], s_vh[tt][j], dkh);
            }
            // dvhat_j = sum_i dS_ij khat_i : warp shuffles, then across warps
#pragma unroll
            for (int j = 0; j < DV; ++j) {
                float x = ds[j] * kh;
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                x += __shfl_xor_sync(0xffffffffu, x, 1);
                if (lane == 0) s_red[warp][j] = x;
            }
            da += qdq_bh[off] - kh * dkh;
            const float dah = kk * dkh;
            const float dah_dg = ta == 0.0f ? 0.0f : ta * exp2f((ta - 1.0f) * log2f(gg));
            const float dah_dtau = ah == 0.0f ? 0.0f : ah * logf(gg);
            if (act) {
                stf(dk_ + off, ah * dkh);
                stf(dg + off, cg * (-ta * da + dah_dg * dah));
                stf(dtau + off, ct * (-gg * da + dah_dtau * dah));
            }
            a_next = al;
            __syncthreads();
            for (int j = threadIdx.x; j < DV; j += blockDim.x) {
                float dvh = 0.0f;
                for (int w = 0; w < nwarps; ++w) dvh += s_red[w][j];
                const size_t ov = (size_t)(t0 + tt) * DV + j;
                const float b_in = ldf(beta + ov);
                const float bb = p.preact ? sigmoid_acc(b_in) : b_in;
                const float df = p.dfeed ? p.dfeed[(size_t)(bh % p.H) * DV + j] * ldf(dO + ov) : 0.0f;
                stf(dv_ + ov, fmaf(bb, dvh, df));
                stf(dbeta + ov, (p.preact ? bb * (1.0f - bb) : 1.0f) * ldf(v + ov) * dvh);
            }
            __syncthreads();
        }
    }
    if (act && p.dS0) {
#pragma unroll
        for (int j = 0; j < DV; ++j) p.dS0[((size_t)bh * dk + i) * DV + j] = a_next * ds[j];
    }
}

template <typename T>
cudaError_t fwd_t(const SeqParams& p, cudaStream_t s) {
    const int grid = p.B * p.H, block = p.dv;
    switch (p.dk) {
        case 16: simt_fwd_kernel<T, 16><<<grid, block, 0, s>>>(p); break;
        case 32: simt_fwd_kernel<T, 32><<<grid, block, 0, s>>>(p); break;
        case 64: simt_fwd_kernel<T, 64><<<grid, block, 0, s>>>(p); break;
        case 128: simt_fwd_kernel<T, 128><<<grid, block, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T, int DV>
cudaError_t bwd_tv(const BwdParams& p, float* qdq, float* fin, const int* only, cudaStream_t s) {
    const int grid = p.B * p.H, block = (p.dk + 31) / 32 * 32;
    simt_bwd_fsweep<T, DV><<<grid, block, 0, s>>>(p, qdq, fin, only);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    simt_bwd_rsweep<T, DV><<<grid, block, 0, s>>>(p, qdq, fin, only);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_t(const BwdParams& p, float* qdq, float* fin, const int* only, cudaStream_t s) {
    switch (p.dv) {
        case 16: return bwd_tv<T, 16>(p, qdq, fin, only, s);
        case 32: return bwd_tv<T, 32>(p, qdq, fin, only, s);
        case 64: return bwd_tv<T, 64>(p, qdq, fin, only, s);
        case 128: return bwd_tv<T, 128>(p, qdq, fin, only, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_simt_fwd(const SeqParams& p, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    return p.bf16 ? fwd_t<__nv_bfloat16>(p, s) : fwd_t<float>(p, s);
}

// scratch: q*dq for every (b,h,t,i) and the final-state term per (b,h,i), float32
size_t simt_bwd_workspace(const BwdParams& p) {
    const size_t rows = (size_t)p.B * p.H * p.dk;
    const size_t a = ((rows * (size_t)p.T * 4) + 255) / 256 * 256;
    return a + rows * 4;
}

static cudaError_t simt_bwd(const BwdParams& p, const int* only, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    const size_t rows = (size_t)p.B * p.H * p.dk;
    const size_t a = ((rows * (size_t)p.T * 4) + 255) / 256 * 256;
    float* qdq = static_cast<float*>(p.ws);
    float* fin = reinterpret_cast<float*>(static_cast<char*>(p.ws) + a);
    return p.bf16 ? bwd_t<__nv_bfloat16>(p, qdq, fin, only, s) : bwd_t<float>(p, qdq, fin, only, s);
}

cudaError_t launch_simt_bwd(const BwdParams& p, cudaStream_t s) { return simt_bwd(p, nullptr, s); }

cudaError_t launch_simt_bwd_flagged(const BwdParams& p, const int* flags, cudaStream_t s) {
    return simt_bwd(p, flags, s);
}

}  // namespace rdm
