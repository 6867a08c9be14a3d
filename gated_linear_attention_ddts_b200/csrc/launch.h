// launch.h -- internal host launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace rdm {

// Default bound of every on-device wait (mbarrier phases, role barriers, flags
// set by other CTAs): about one second of SM clock cycles.
constexpr long long kDefaultWaitLimit = 2000000000LL;

struct SeqParams {
    int B, H, T, dk, dv, chunk;
    int bf16;    // element type of sequence tensors: 1 = bf16, 0 = float32
    int preact;  // g, tau, beta are pre-activations (softplus, sigmoid, sigmoid applied inside)
    const void *q, *k, *v, *g, *tau, *beta;
    const float* S0;
    void* o;
    float* ST;
    float* saved;        // [B,H,NC,dk,dv] chunk-start states, or null
    void* ws;            // scratch for sequence segments, or null
    size_t ws_bytes;
    unsigned* err;       // device status word
    long long wait_limit;  // SM clock cycles a bounded wait may take before it gives up
    int withhold_flags;    // test hook: segment CTAs never publish their flags
    const float* dfeed;    // feedthrough weights [H][dv]: o_t += d (.) v_t; null = none
    // low-rank beta_hat (preact only): pre-activation u[b,t,:] . w_up[h][:, j],
    // u [B,T,beta_rank] bf16, w_up [H,beta_rank,dv] float32; beta unused.  0 = off
    int beta_rank;
    const void* beta_u;
    const float* beta_w;
};

struct BwdParams {
    int B, H, T, dk, dv, chunk;
    int bf16;
    int preact;  // as SeqParams::preact; grad_g, grad_tau, grad_beta then refer to the pre-activations
    const void *q, *k, *v, *g, *tau, *beta;
    const float* S0;
    const void* dO;
    const float* dST;
    const float* saved;  // chunk-start states (tensor-core path), or null
    void *dq, *dk_, *dv_, *dg, *dtau, *dbeta;
    float* dS0;
    void* ws;            // scratch
    size_t ws_bytes;
    unsigned* err;
    long long wait_limit;  // as SeqParams
    int withhold_flags;
    const float* dfeed;    // feedthrough weights [H][dv], or null
    float* grad_dfeed;     // dL/d(feedthrough) [H][dv], written when non-null
};

struct DecodeParams {
    int B, H, dk, dv;
    int bf16;
    const void *q, *k, *v, *g, *tau, *beta;
    float* S;
    void* o;
    const float* dfeed;  // feedthrough weights [H][dv], or null
};

// exact token-serial CUDA-core path (any supported shape, float32 or bf16)
cudaError_t launch_simt_fwd(const SeqParams& p, cudaStream_t s);
size_t simt_bwd_workspace(const BwdParams& p);
cudaError_t launch_simt_bwd(const BwdParams& p, cudaStream_t s);
// same, for the heads with flags[b*H + h] != 0 only (the others return at once)
cudaError_t launch_simt_bwd_flagged(const BwdParams& p, const int* flags, cudaStream_t s);

// decode step
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s);

// ShortConv: causal depthwise convolution along the tokens (shortconv.cu)
struct ConvParams {
    int B, H, T, D, W;
    int bf16;   // element type of x, y, states and their gradients
    int silu;   // y = z * sigmoid(z) instead of y = z
    const void* x;       // [B,H,T,D]
    const float* w;      // [H,D,W]
    const float* bias;   // [H,D] or null
    const void* xs;      // carried-in state [B,H,W-1,D] or null (zeros)
    void* y;             // [B,H,T,D]
    void* xs_out;        // carried-out state [B,H,W-1,D] or null
    const void* dy;      // backward: dL/dy
    const void* dxs_out; // dL/d(carried-out state) or null
    void* dx;            // dL/dx
    float* dw;           // dL/dw [H,D,W]
    float* dbias;        // dL/dbias [H,D] or null
    void* dxs;           // dL/d(carried-in state) or null
    int tile;            // tokens per block (set by the launcher)
    unsigned* err;       // device status word (a staging wait that ran out)
    long long wait_limit;
    int withhold;        // test hook: the staging copies are never issued
};
cudaError_t launch_conv_fwd(const ConvParams& p, cudaStream_t s);
cudaError_t launch_conv_bwd(const ConvParams& p, cudaStream_t s);

// gradient of the feedthrough weights: grad_d[h][j] = sum_{b,t} dO[b,h,t,j] v[b,h,t,j]
// (zeroes grad_d, then accumulates; float32 atomics)
cudaError_t launch_feed_grad(const BwdParams& p, cudaStream_t s);

// low-rank beta_hat (lowrank.cu): expansion of the pre-activation for the
// backward, and the contraction of its gradient
struct LowRankParams {
    int B, H, T, dv, r;
    int bf16;                // element type of u, beta_pre, dbeta_pre, du
    const void* u;           // [B,T,r]
    const float* w;          // [H,r,dv]
    void* beta_pre;          // [B,H,T,dv] written by the expansion
    const void* dbeta_pre;   // [B,H,T,dv] gradient w.r.t. the pre-activation
    void* du;                // [B,T,r]
    float* dw;               // [H,r,dv]
};
cudaError_t launch_lowrank_expand(const LowRankParams& p, cudaStream_t s);
cudaError_t launch_lowrank_grad(const LowRankParams& p, cudaStream_t s);

// tensor-core (tcgen05) chunked path
bool tc_fwd_supported(const SeqParams& p);
size_t tc_fwd_workspace(const SeqParams& p);  // bytes that enable sequence segments
cudaError_t launch_tc_fwd(const SeqParams& p, cudaStream_t s);
bool tc_bwd_supported(const BwdParams& p);
size_t tc_bwd_workspace(const BwdParams& p);
cudaError_t launch_tc_bwd(const BwdParams& p, cudaStream_t s);

}  // namespace rdm

// ---------------------------------------------------------------- TMA maps
#include <cuda.h>
namespace rdm {
// 3-D bf16 tensor [n2][n1][n0] (n0 innermost, dense) as a TMA map with box
// {b0, b1, 1} and 128-byte swizzle (b0 * 2 must be 128).  Returns false if the
// driver refuses the map.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1,
                       uint64_t n2, uint32_t b0, uint32_t b1);

// The same without swizzle (rows of the box land b0 * 2 bytes apart); b0 * 2
// a multiple of 16.
bool make_tmap_bf16_3d_plain(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1,
                             uint64_t n2, uint32_t b0, uint32_t b1);

// 2-D float32 tensor [n1][n0] (n0 innermost, dense) as a TMA map with box
// {b0, b1} and 128-byte swizzle (b0 * 4 must be 128).
bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint32_t b0,
                      uint32_t b1);

// SM count of the current device (cached).
int sm_count();
// Tag of one launch for flags that CTAs of a sequence-segmented kernel set for
// one another: distinct for every launch of the process, seeded from the clock
// so that it is unlikely to equal what a reused workspace still holds.
unsigned next_launch_tag();
}  // namespace rdm
