// decode.cu -- one token of sequential DDTS inference on a cached float32
// state (Rodimus*, paperhub.cn rebuttal Q2: sequential inference on a
// fixed-size hidden state, O(1) per token).  For every (b,h):
//     S <- diag(alpha) S + (alpha_hat*k)(beta_hat*v)^T ;  o = S^T q
//
// The step is a pure stream of the state: 2 * d_k * d_v * 4 bytes per (b,h)
// against a few hundred bytes of token inputs.  One 128-thread block owns one
// (b,h); each thread owns 4 adjacent columns (one float4) of every
// (128 / (d_v/4))-th row, so a warp reads/writes whole 512-byte row segments
// and the q-reduction for o stays inside the thread until one shared-memory
// pass at the end.
#include "launch.h"
#include "rdm_common.cuh"

namespace rdm {
namespace {

constexpr int kThreads = 128;
constexpr int kBatch = 8;  // rows loaded before any is written back

template <typename T, int DV>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeParams p) {
    constexpr int CQ = DV / 4;        // float4 column groups per row
    constexpr int RS = kThreads / CQ;  // rows processed concurrently
    const int bh = blockIdx.x;
    const int dk = p.dk;
    __shared__ float s_al[128], s_kh[128], s_q[128];
    __shared__ float4 s_red[RS][CQ];

    const T* q = static_cast<const T*>(p.q) + (size_t)bh * dk;
    const T* k = static_cast<const T*>(p.k) + (size_t)bh * dk;
    const T* g = static_cast<const T*>(p.g) + (size_t)bh * dk;
    const T* tau = static_cast<const T*>(p.tau) + (size_t)bh * dk;
    const T* v = static_cast<const T*>(p.v) + (size_t)bh * DV;
    const T* beta = static_cast<const T*>(p.beta) + (size_t)bh * DV;

    for (int i = threadIdx.x; i < dk; i += kThreads) {
        const float gg = ldf(g + i), tt = ldf(tau + i);
        s_al[i] = alpha(gg, tt);
        s_kh[i] = alpha_hat(gg, tt) * ldf(k + i);
        s_q[i] = ldf(q + i);
    }
    const int cq = threadIdx.x % CQ, rs = threadIdx.x / CQ;
    float vh[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) vh[c] = ldf(beta + 4 * cq + c) * ldf(v + 4 * cq + c);
    __syncthreads();

    float4* S = reinterpret_cast<float4*>(p.S + (size_t)bh * dk * DV) + cq;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = rs; i0 < dk; i0 += RS * kBatch) {
        float4 s[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * RS;
            if (i < dk) s[u] = S[(size_t)i * CQ];
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * RS;
            if (i < dk) {
                const float a = s_al[i], kk = s_kh[i], qi = s_q[i];
                s[u].x = fmaf(a, s[u].x, kk * vh[0]);
                s[u].y = fmaf(a, s[u].y, kk * vh[1]);
                s[u].z = fmaf(a, s[u].z, kk * vh[2]);
                s[u].w = fmaf(a, s[u].w, kk * vh[3]);
                S[(size_t)i * CQ] = s[u];
                acc.x = fmaf(qi, s[u].x, acc.x);
                acc.y = fmaf(qi, s[u].y, acc.y);
                acc.z = fmaf(qi, s[u].z, acc.z);
                acc.w = fmaf(qi, s[u].w, acc.w);
            }
        }
    }
    s_red[rs][cq] = acc;
    __syncthreads();
    if (rs == 0) {
        float4 o4 = s_red[0][cq];
        if (p.dfeed) {  // feedthrough o += d (.) v
            const float* d = p.dfeed + (size_t)(bh % p.H) * DV + 4 * cq;
            o4.x = fmaf(d[0], ldf(v + 4 * cq + 0), o4.x);
            o4.y = fmaf(d[1], ldf(v + 4 * cq + 1), o4.y);
            o4.z = fmaf(d[2], ldf(v + 4 * cq + 2), o4.z);
            o4.w = fmaf(d[3], ldf(v + 4 * cq + 3), o4.w);
        }
#pragma unroll
        for (int r = 1; r < RS; ++r) {
            const float4 x = s_red[r][cq];
            o4.x += x.x; o4.y += x.y; o4.z += x.z; o4.w += x.w;
        }
        T* o = static_cast<T*>(p.o) + (size_t)bh * DV + 4 * cq;
        stf(o + 0, o4.x);
        stf(o + 1, o4.y);
        stf(o + 2, o4.z);
        stf(o + 3, o4.w);
    }
}

template <typename T>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
    const int grid = p.B * p.H;
    switch (p.dv) {
        case 16: decode_kernel<T, 16><<<grid, kThreads, 0, s>>>(p); break;
        case 32: decode_kernel<T, 32><<<grid, kThreads, 0, s>>>(p); break;
        case 64: decode_kernel<T, 64><<<grid, kThreads, 0, s>>>(p); break;
        case 128: decode_kernel<T, 128><<<grid, kThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
    return p.bf16 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace rdm
