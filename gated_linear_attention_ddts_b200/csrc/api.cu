// api.cu -- the exported C ABI (include/rdm_ddts.h): argument validation,
// path selection and launch.  Nothing here allocates device memory or
// synchronises, except rdm_ddts_sync_status.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/rdm_ddts.h"
#include "conv_launch.h"
#include "launch.h"
#include "rdm_common.cuh"
#include "ska_launch.h"

namespace rdm {

// Device status word (bit kErrTimeout: a bounded wait ran out).  One copy per
// device the library is loaded on.
__device__ unsigned g_status_word;

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_status_ptr[kMaxDevices];

unsigned* status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_status_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<unsigned*>(ptr);
    }
    return g_status_ptr[dev];
}

// Test hooks (rdm_ddts_set_test_hooks): a shorter bound for on-device waits and
// segment flags that are never published; 0 = off.
std::atomic<long long> g_hook_wait_limit{0};
std::atomic<int> g_hook_withhold{0};

long long wait_limit() {
    const long long w = g_hook_wait_limit.load(std::memory_order_relaxed);
    return w > 0 ? w : kDefaultWaitLimit;
}

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool opt_aligned(const void* p) { return p == nullptr || aligned(p); }

rdm_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RDM_OK : RDM_ERR_CUDA; }

// Sizes shared by fwd and bwd.  Returns RDM_OK or the reason to refuse.
rdm_status check_sizes(int B, int H, int T, int dk, int dv, int chunk, rdm_dtype dtype,
                       rdm_impl impl) {
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return RDM_ERR_INVALID_ARG;
    if (dtype != RDM_F32 && dtype != RDM_BF16) return RDM_ERR_INVALID_ARG;
    if (impl != RDM_IMPL_AUTO && impl != RDM_IMPL_SIMT && impl != RDM_IMPL_TC)
        return RDM_ERR_INVALID_ARG;
    if (chunk < 0) return RDM_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return RDM_ERR_UNSUPPORTED;
    if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128)
        return RDM_ERR_UNSUPPORTED;
    // every element offset must fit in 63 bits and the grid in 31
    const double n = (double)B * H * (double)(T > 0 ? T : 1) * (dk > dv ? dk : dv);
    if (n > 4.0e18 || (double)B * H > 2.0e9 || T > (1 << 30)) return RDM_ERR_INVALID_ARG;
    return RDM_OK;
}

int eff_chunk(int chunk) { return chunk == 0 ? 64 : chunk; }

bool gates_ok(rdm_gate_inputs g) { return g == RDM_GATES_ACTIVATED || g == RDM_GATES_PREACT; }

// T == 0: no tokens; S_T = S_0 (or zero), no saved states.
rdm_status empty_sequence(int B, int H, int dk, int dv, const float* S0, float* ST,
                          cudaStream_t s) {
    if (!ST) return RDM_OK;
    const size_t bytes = (size_t)B * H * dk * dv * 4;
    cudaError_t e = S0 ? cudaMemcpyAsync(ST, S0, bytes, cudaMemcpyDeviceToDevice, s)
                       : cudaMemsetAsync(ST, 0, bytes, s);
    return from_cuda(e);
}

bool use_tc_fwd(const SeqParams& p, rdm_impl impl) {
    if (impl == RDM_IMPL_SIMT) return false;
    return tc_fwd_supported(p);
}

bool use_tc_bwd(const BwdParams& p, rdm_impl impl) {
    if (impl == RDM_IMPL_SIMT) return false;
    return tc_bwd_supported(p);
}

SeqParams fwd_params(const rdm_fwd_args* a) {
    SeqParams p;
    memset(&p, 0, sizeof(p));
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv;
    p.chunk = eff_chunk(a->chunk);
    p.bf16 = a->dtype == RDM_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.tau = a->tau; p.beta = a->beta;
    p.S0 = a->S0; p.o = a->o; p.ST = a->ST; p.saved = a->saved_states;
    p.ws = a->workspace; p.ws_bytes = a->workspace ? a->workspace_bytes : 0;
    p.preact = a->gate_inputs == RDM_GATES_PREACT;
    p.wait_limit = wait_limit();
    p.withhold_flags = g_hook_withhold.load(std::memory_order_relaxed);
    p.dfeed = a->feedthrough;
    p.beta_rank = a->beta_rank;
    p.beta_u = a->beta_u;
    p.beta_w = a->beta_w;
    return p;
}

// Low-rank beta_hat arguments (beta_rank > 0): rank 8 or 16, the factors given
// and aligned, gates passed as pre-activations.
rdm_status check_lowrank(int rank, const void* u, const float* w, rdm_gate_inputs g) {
    if (rank == 0) return RDM_OK;
    if (rank < 0) return RDM_ERR_INVALID_ARG;
    if (rank != 8 && rank != 16) return RDM_ERR_UNSUPPORTED;
    if (g != RDM_GATES_PREACT || !u || !w || !aligned(u) || !aligned(w)) return RDM_ERR_INVALID_ARG;
    return RDM_OK;
}

size_t lowrank_buffer_bytes(int B, int H, int T, int dv, rdm_dtype dt) {
    const size_t n = (size_t)B * H * T * dv * (dt == RDM_BF16 ? 2 : 4);
    return (n + 255) / 256 * 256;
}

BwdParams bwd_params(const rdm_bwd_args* a) {
    BwdParams p;
    memset(&p, 0, sizeof(p));
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv;
    p.chunk = eff_chunk(a->chunk);
    p.bf16 = a->dtype == RDM_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.tau = a->tau; p.beta = a->beta;
    p.S0 = a->S0; p.dO = a->grad_o; p.dST = a->grad_ST; p.saved = a->saved_states;
    p.dq = a->grad_q; p.dk_ = a->grad_k; p.dv_ = a->grad_v; p.dg = a->grad_g;
    p.dtau = a->grad_tau; p.dbeta = a->grad_beta; p.dS0 = a->grad_S0;
    p.ws = a->workspace; p.ws_bytes = a->workspace_bytes;
    p.preact = a->gate_inputs == RDM_GATES_PREACT;
    p.wait_limit = wait_limit();
    p.withhold_flags = g_hook_withhold.load(std::memory_order_relaxed);
    p.dfeed = a->feedthrough;
    p.grad_dfeed = a->grad_feedthrough;
    return p;
}

}  // namespace
}  // namespace rdm

using namespace rdm;

extern "C" {

size_t rdm_ddts_saved_states_size(int B, int H, int T, int dk, int dv, int chunk) {
    if (check_sizes(B, H, T, dk, dv, chunk, RDM_F32, RDM_IMPL_AUTO) != RDM_OK) return 0;
    const int C = eff_chunk(chunk);
    const size_t nc = (size_t)(T + C - 1) / C;
    return (size_t)B * H * nc * dk * dv * 4;
}

rdm_status rdm_ddts_fwd(const rdm_fwd_args* a, rdm_stream_t stream) {
    if (!a) return RDM_ERR_INVALID_ARG;
    rdm_status st = check_sizes(a->B, a->H, a->T, a->dk, a->dv, a->chunk, a->dtype, a->impl);
    if (st != RDM_OK) return st;
    if (!gates_ok(a->gate_inputs)) return RDM_ERR_INVALID_ARG;
    st = check_lowrank(a->beta_rank, a->beta_u, a->beta_w, a->gate_inputs);
    if (st != RDM_OK) return st;
    const bool lr = a->beta_rank > 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!opt_aligned(a->S0) || !opt_aligned(a->ST) || !opt_aligned(a->saved_states) ||
        !opt_aligned(a->workspace) || !opt_aligned(a->feedthrough))
        return RDM_ERR_INVALID_ARG;
    if (a->T == 0) {
        if ((a->impl == RDM_IMPL_TC || lr) && a->dtype != RDM_BF16) return RDM_ERR_UNSUPPORTED;
        return empty_sequence(a->B, a->H, a->dk, a->dv, a->S0, a->ST, s);
    }
    const void* in[] = {a->q, a->k, a->v, a->g, a->tau, lr ? a->v : a->beta, a->o};
    for (const void* p : in)
        if (!p || !aligned(p)) return RDM_ERR_INVALID_ARG;
    SeqParams p = fwd_params(a);
    p.err = status_word();
    if (!p.err) return RDM_ERR_CUDA;
    const bool tc = use_tc_fwd(p, a->impl);
    if ((a->impl == RDM_IMPL_TC || lr) && !tc) return RDM_ERR_UNSUPPORTED;
    return from_cuda(tc ? launch_tc_fwd(p, s) : launch_simt_fwd(p, s));
}

size_t rdm_ddts_fwd_workspace_size(const rdm_fwd_args* a) {
    if (!a) return (size_t)-1;
    if (check_sizes(a->B, a->H, a->T, a->dk, a->dv, a->chunk, a->dtype, a->impl) != RDM_OK ||
        !gates_ok(a->gate_inputs) ||
        check_lowrank(a->beta_rank, a->beta_u, a->beta_w, a->gate_inputs) == RDM_ERR_INVALID_ARG)
        return (size_t)-1;
    if (a->T == 0) return 0;
    SeqParams p = fwd_params(a);
    return use_tc_fwd(p, a->impl) ? tc_fwd_workspace(p) : 0;
}

size_t rdm_ddts_bwd_workspace_size(const rdm_bwd_args* a) {
    if (!a) return (size_t)-1;
    if (check_sizes(a->B, a->H, a->T, a->dk, a->dv, a->chunk, a->dtype, a->impl) != RDM_OK ||
        !gates_ok(a->gate_inputs))
        return (size_t)-1;
    if (check_lowrank(a->beta_rank, a->beta_u, a->beta_w, a->gate_inputs) == RDM_ERR_INVALID_ARG)
        return (size_t)-1;
    if (a->T == 0) return 0;
    BwdParams p = bwd_params(a);
    const size_t base = use_tc_bwd(p, a->impl) ? tc_bwd_workspace(p) : simt_bwd_workspace(p);
    if (a->beta_rank <= 0) return base;
    // the expanded pre-activation and its gradient follow the kernels' scratch
    return (base + 255) / 256 * 256 + 2 * lowrank_buffer_bytes(a->B, a->H, a->T, a->dv, a->dtype);
}

rdm_status rdm_ddts_bwd(const rdm_bwd_args* a, rdm_stream_t stream) {
    if (!a) return RDM_ERR_INVALID_ARG;
    rdm_status st = check_sizes(a->B, a->H, a->T, a->dk, a->dv, a->chunk, a->dtype, a->impl);
    if (st != RDM_OK) return st;
    if (!gates_ok(a->gate_inputs)) return RDM_ERR_INVALID_ARG;
    st = check_lowrank(a->beta_rank, a->beta_u, a->beta_w, a->gate_inputs);
    if (st != RDM_OK) return st;
    const bool lr = a->beta_rank > 0;
    if (lr && (!a->grad_beta_u || !a->grad_beta_w || !aligned(a->grad_beta_u) ||
               !aligned(a->grad_beta_w)))
        return RDM_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!opt_aligned(a->S0) || !opt_aligned(a->grad_ST) || !opt_aligned(a->grad_S0) ||
        !opt_aligned(a->saved_states) || !opt_aligned(a->workspace) ||
        !opt_aligned(a->feedthrough) || !opt_aligned(a->grad_feedthrough))
        return RDM_ERR_INVALID_ARG;
    if (a->grad_feedthrough && !a->feedthrough) return RDM_ERR_INVALID_ARG;
    if (a->T == 0) {
        if (a->impl == RDM_IMPL_TC && a->dtype != RDM_BF16) return RDM_ERR_UNSUPPORTED;
        // no tokens: dS_0 = dS_T, and the feedthrough gradient is zero
        if (a->grad_feedthrough &&
            cudaMemsetAsync(a->grad_feedthrough, 0, (size_t)a->H * a->dv * 4, s) != cudaSuccess)
            return RDM_ERR_CUDA;
        if (lr && cudaMemsetAsync(a->grad_beta_w, 0, (size_t)a->H * a->beta_rank * a->dv * 4, s) !=
                      cudaSuccess)
            return RDM_ERR_CUDA;
        return empty_sequence(a->B, a->H, a->dk, a->dv, a->grad_ST, a->grad_S0, s);
    }
    const void* in[] = {a->q, a->k, a->v, a->g, a->tau, lr ? a->v : a->beta, a->grad_o, a->grad_q,
                        a->grad_k, a->grad_v, a->grad_g, a->grad_tau,
                        lr ? a->grad_v : a->grad_beta};
    for (const void* p : in)
        if (!p || !aligned(p)) return RDM_ERR_INVALID_ARG;
    BwdParams p = bwd_params(a);
    p.err = status_word();
    if (!p.err) return RDM_ERR_CUDA;
    const bool tc = use_tc_bwd(p, a->impl);
    if (a->impl == RDM_IMPL_TC && !tc) return RDM_ERR_UNSUPPORTED;
    const size_t base = tc ? tc_bwd_workspace(p) : simt_bwd_workspace(p);
    const size_t lrb = lr ? lowrank_buffer_bytes(a->B, a->H, a->T, a->dv, a->dtype) : 0;
    const size_t need = lr ? (base + 255) / 256 * 256 + 2 * lrb : base;
    if (need > 0 && (!a->workspace || a->workspace_bytes < need)) return RDM_ERR_WORKSPACE;
    LowRankParams lp{};
    if (lr) {
        // beta_pre = u . w_up into the workspace, its gradient beside it
        uint8_t* ws = static_cast<uint8_t*>(a->workspace) + (base + 255) / 256 * 256;
        lp.B = a->B; lp.H = a->H; lp.T = a->T; lp.dv = a->dv; lp.r = a->beta_rank;
        lp.bf16 = a->dtype == RDM_BF16;
        lp.u = a->beta_u; lp.w = a->beta_w;
        lp.beta_pre = ws; lp.dbeta_pre = ws + lrb;
        lp.du = a->grad_beta_u; lp.dw = a->grad_beta_w;
        p.beta = lp.beta_pre;
        p.dbeta = ws + lrb;
        p.ws_bytes = base;
        cudaError_t e = launch_lowrank_expand(lp, s);
        if (e != cudaSuccess) return from_cuda(e);
    }
    cudaError_t e = tc ? launch_tc_bwd(p, s) : launch_simt_bwd(p, s);
    if (e == cudaSuccess && p.grad_dfeed) e = launch_feed_grad(p, s);
    if (e == cudaSuccess && lr) e = launch_lowrank_grad(lp, s);
    return from_cuda(e);
}

rdm_status rdm_ddts_decode(const rdm_decode_args* a, rdm_stream_t stream) {
    if (!a) return RDM_ERR_INVALID_ARG;
    rdm_status st = check_sizes(a->B, a->H, 1, a->dk, a->dv, 0, a->dtype, RDM_IMPL_AUTO);
    if (st != RDM_OK) return st;
    const void* in[] = {a->q, a->k, a->v, a->g, a->tau, a->beta, a->S, a->o};
    for (const void* p : in)
        if (!p || !aligned(p)) return RDM_ERR_INVALID_ARG;
    if (!opt_aligned(a->feedthrough)) return RDM_ERR_INVALID_ARG;
    DecodeParams p;
    p.B = a->B; p.H = a->H; p.dk = a->dk; p.dv = a->dv; p.bf16 = a->dtype == RDM_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.tau = a->tau; p.beta = a->beta;
    p.S = a->S; p.o = a->o; p.dfeed = a->feedthrough;
    return from_cuda(launch_decode(p, reinterpret_cast<cudaStream_t>(stream)));
}

rdm_status rdm_ddts_decode_step(int B, int H, int dk, int dv, rdm_dtype dtype, const void* q,
                                const void* k, const void* v, const void* g, const void* tau,
                                const void* beta, float* S, void* o, rdm_stream_t stream) {
    rdm_decode_args a;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv; a.dtype = dtype;
    a.q = q; a.k = k; a.v = v; a.g = g; a.tau = tau; a.beta = beta; a.S = S; a.o = o;
    a.feedthrough = nullptr;
    return rdm_ddts_decode(&a, stream);
}

static rdm_status conv_check(const rdm_shortconv_args* a) {
    if (!a || a->B < 1 || a->H < 1 || a->T < 0 || a->W < 1) return RDM_ERR_INVALID_ARG;
    if (a->dtype != RDM_F32 && a->dtype != RDM_BF16) return RDM_ERR_INVALID_ARG;
    if (!(a->D == 16 || a->D == 32 || a->D == 64 || a->D == 128) || a->W > 4) return RDM_ERR_UNSUPPORTED;
    if ((double)a->B * a->H * (double)(a->T > 0 ? a->T : 1) * a->D > 4.0e18 || (double)a->B * a->H > 2.0e9)
        return RDM_ERR_INVALID_ARG;
    if (!a->weight || !aligned(a->weight) || !opt_aligned(a->bias) || !opt_aligned(a->state_in))
        return RDM_ERR_INVALID_ARG;
    if (a->T > 0 && (!a->x || !aligned(a->x))) return RDM_ERR_INVALID_ARG;
    return RDM_OK;
}

static ConvParams conv_params(const rdm_shortconv_args* a) {
    ConvParams p;
    memset(&p, 0, sizeof(p));
    p.B = a->B; p.H = a->H; p.T = a->T; p.D = a->D; p.W = a->W;
    p.bf16 = a->dtype == RDM_BF16;
    p.silu = a->silu != 0;
    p.x = a->x; p.w = a->weight; p.bias = a->bias; p.xs = a->state_in;
    p.y = a->y; p.xs_out = a->W > 1 ? a->state_out : nullptr;
    p.err = status_word();
    p.wait_limit = wait_limit();
    p.withhold = g_hook_withhold.load(std::memory_order_relaxed);
    return p;
}

// argument checks of one problem (no CUDA call)
static rdm_status conv_fwd_check(const rdm_shortconv_args* a) {
    rdm_status st = conv_check(a);
    if (st != RDM_OK) return st;
    if (a->T > 0 && (!a->y || !aligned(a->y))) return RDM_ERR_INVALID_ARG;
    if (!opt_aligned(a->state_out)) return RDM_ERR_INVALID_ARG;
    return RDM_OK;
}

static rdm_status conv_bwd_check(const rdm_shortconv_bwd_args* a) {
    rdm_status st = conv_check(&a->fwd);
    if (st != RDM_OK) return st;
    if (!a->grad_weight || !aligned(a->grad_weight) || !opt_aligned(a->grad_bias) ||
        !opt_aligned(a->grad_state_in) || !opt_aligned(a->grad_state_out))
        return RDM_ERR_INVALID_ARG;
    if (a->fwd.T > 0 && (!a->grad_y || !aligned(a->grad_y) || !a->grad_x || !aligned(a->grad_x)))
        return RDM_ERR_INVALID_ARG;
    return RDM_OK;
}

static rdm_status conv_bwd_params(const rdm_shortconv_bwd_args* a, ConvParams* p) {
    *p = conv_params(&a->fwd);
    if (!p->err) return RDM_ERR_CUDA;
    p->y = nullptr;
    p->xs_out = nullptr;
    p->dy = a->grad_y;
    p->dxs_out = a->fwd.W > 1 ? a->grad_state_out : nullptr;
    p->dx = a->grad_x;
    p->dw = a->grad_weight;
    p->dbias = a->fwd.bias ? a->grad_bias : nullptr;
    p->dxs = (a->fwd.state_in && a->fwd.W > 1) ? a->grad_state_in : nullptr;
    return RDM_OK;
}

// one launch serves problems of the same element type, width and activation
static bool conv_same_kind(const rdm_shortconv_args& a, const rdm_shortconv_args& b) {
    return a.dtype == b.dtype && a.W == b.W && (a.silu != 0) == (b.silu != 0);
}

rdm_status rdm_shortconv_fwd(const rdm_shortconv_args* a, rdm_stream_t stream) {
    return rdm_shortconv_fwd_many(a, 1, stream);
}

rdm_status rdm_shortconv_bwd(const rdm_shortconv_bwd_args* a, rdm_stream_t stream) {
    return rdm_shortconv_bwd_many(a, 1, stream);
}

rdm_status rdm_shortconv_fwd_many(const rdm_shortconv_args* a, int n, rdm_stream_t stream) {
    if (!a || n < 1 || n > kMaxConvBatch) return RDM_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (!conv_same_kind(a[0], a[i])) return RDM_ERR_INVALID_ARG;
        rdm_status st = conv_fwd_check(&a[i]);
        if (st != RDM_OK) return st;
    }
    ConvParams ps[kMaxConvBatch];
    for (int i = 0; i < n; ++i) {
        ps[i] = conv_params(&a[i]);
        if (!ps[i].err) return RDM_ERR_CUDA;
    }
    // problems without sequences have nothing to compute
    int m = 0;
    for (int i = 0; i < n; ++i)
        if (ps[i].B * ps[i].H > 0) ps[m++] = ps[i];
    if (m == 0) return RDM_OK;
    return from_cuda(launch_conv_fwd_many(ps, m, reinterpret_cast<cudaStream_t>(stream)));
}

rdm_status rdm_shortconv_bwd_many(const rdm_shortconv_bwd_args* a, int n, rdm_stream_t stream) {
    if (!a || n < 1 || n > kMaxConvBatch) return RDM_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (!conv_same_kind(a[0].fwd, a[i].fwd)) return RDM_ERR_INVALID_ARG;
        rdm_status st = conv_bwd_check(&a[i]);
        if (st != RDM_OK) return st;
    }
    ConvParams ps[kMaxConvBatch];
    for (int i = 0; i < n; ++i) {
        rdm_status st = conv_bwd_params(&a[i], &ps[i]);
        if (st != RDM_OK) return st;
    }
    return from_cuda(launch_conv_bwd_many(ps, n, reinterpret_cast<cudaStream_t>(stream)));
}

static bool ska_dim_ok(int d) { return d == 64 || d == 128; }

static float ska_scale(float scale, int dk) {
    return scale == 0.0f ? 1.0f / sqrtf((float)dk) : scale;
}

rdm_status rdm_ska_fwd(const rdm_ska_fwd_args* a, rdm_stream_t stream) {
    if (!a || a->B < 1 || a->H < 1 || a->T < 0 || a->window < 1) return RDM_ERR_INVALID_ARG;
    if (!(a->scale >= 0.0f) || isinf(a->scale)) return RDM_ERR_INVALID_ARG;
    if (a->dtype != RDM_BF16) return a->dtype == RDM_F32 ? RDM_ERR_UNSUPPORTED : RDM_ERR_INVALID_ARG;
    if (!ska_dim_ok(a->dk) || !ska_dim_ok(a->dv)) return RDM_ERR_UNSUPPORTED;
    if ((double)a->B * a->H * ((a->T + 127) / 128) > 2.0e9 || a->T > (1 << 30))
        return RDM_ERR_INVALID_ARG;
    if (a->T > 0 && (!a->q || !a->k || !a->v || !a->o)) return RDM_ERR_INVALID_ARG;
    if (!opt_aligned(a->q) || !opt_aligned(a->k) || !opt_aligned(a->v) || !opt_aligned(a->o) ||
        !opt_aligned(a->k_cache) || !opt_aligned(a->v_cache) ||
        (reinterpret_cast<uintptr_t>(a->pos) & 3u) != 0)
        return RDM_ERR_INVALID_ARG;
    if (a->T > 0 && ((a->k_cache && !a->k) || (a->v_cache && !a->v))) return RDM_ERR_INVALID_ARG;
    unsigned* err = status_word();
    if (!err) return RDM_ERR_CUDA;
    SkaParams p;
    memset(&p, 0, sizeof(p));
    p.B = a->B; p.H = a->H; p.T = a->T; p.dk = a->dk; p.dv = a->dv; p.window = a->window;
    p.scale = ska_scale(a->scale, a->dk);
    p.q = a->q; p.k = a->k; p.v = a->v; p.o = a->o;
    p.k_cache = a->T > 0 ? a->k_cache : nullptr;
    p.v_cache = a->T > 0 ? a->v_cache : nullptr;
    p.pos = a->pos;
    p.err = err;
    p.wait_limit = wait_limit();
    p.withhold = g_hook_withhold.load(std::memory_order_relaxed);
    return from_cuda(launch_ska_fwd(p, static_cast<cudaStream_t>(stream)));
}

rdm_status rdm_ska_decode(const rdm_ska_decode_args* a, rdm_stream_t stream) {
    if (!a || a->B < 1 || a->H < 1 || a->window < 1 || a->window > 32768) return RDM_ERR_INVALID_ARG;
    if (!(a->scale >= 0.0f) || isinf(a->scale)) return RDM_ERR_INVALID_ARG;
    if (a->dtype != RDM_BF16) return a->dtype == RDM_F32 ? RDM_ERR_UNSUPPORTED : RDM_ERR_INVALID_ARG;
    if (!ska_dim_ok(a->dk) || !ska_dim_ok(a->dv)) return RDM_ERR_UNSUPPORTED;
    if ((double)a->B * a->H > 2.0e9) return RDM_ERR_INVALID_ARG;
    if (!a->q || !a->k || !a->v || !a->k_cache || !a->v_cache || !a->pos || !a->o)
        return RDM_ERR_INVALID_ARG;
    if (!aligned(a->q) || !aligned(a->k) || !aligned(a->v) || !aligned(a->k_cache) ||
        !aligned(a->v_cache) || !aligned(a->o) || (reinterpret_cast<uintptr_t>(a->pos) & 3u) != 0)
        return RDM_ERR_INVALID_ARG;
    SkaDecodeParams p;
    memset(&p, 0, sizeof(p));
    p.B = a->B; p.H = a->H; p.dk = a->dk; p.dv = a->dv; p.window = a->window;
    p.scale = ska_scale(a->scale, a->dk);
    p.q = a->q; p.k = a->k; p.v = a->v; p.k_cache = a->k_cache; p.v_cache = a->v_cache;
    p.pos = a->pos; p.advance = a->advance_pos != 0; p.o = a->o;
    p.err = status_word();
    if (!p.err) return RDM_ERR_CUDA;
    return from_cuda(launch_ska_decode(p, static_cast<cudaStream_t>(stream)));
}

rdm_status rdm_ddts_sync_status(rdm_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return RDM_ERR_CUDA;
    unsigned* w = status_word();
    if (!w) return RDM_ERR_CUDA;
    unsigned h = 0;
    if (cudaMemcpy(&h, w, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return RDM_ERR_CUDA;
    if (h != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return RDM_ERR_CUDA;
        if (h & kErrTimeout) return RDM_ERR_TIMEOUT;
        if (h & kErrBadValue) return RDM_ERR_INVALID_ARG;
    }
    return RDM_OK;
}

const char* rdm_status_string(rdm_status s) {
    switch (s) {
        case RDM_OK: return "ok";
        case RDM_ERR_INVALID_ARG: return "invalid argument (size, NULL or misaligned pointer)";
        case RDM_ERR_UNSUPPORTED: return "unsupported configuration";
        case RDM_ERR_CUDA: return "CUDA runtime error";
        case RDM_ERR_TIMEOUT: return "a bounded on-device wait timed out";
        case RDM_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

rdm_status rdm_ddts_set_test_hooks(long long wait_limit_cycles, int withhold_segment_flags) {
    if (wait_limit_cycles < 0 || (withhold_segment_flags != 0 && withhold_segment_flags != 1))
        return RDM_ERR_INVALID_ARG;
    g_hook_wait_limit.store(wait_limit_cycles, std::memory_order_relaxed);
    g_hook_withhold.store(withhold_segment_flags, std::memory_order_relaxed);
    return RDM_OK;
}

int rdm_ddts_version(void) { return 700; }

}  // extern "C"
