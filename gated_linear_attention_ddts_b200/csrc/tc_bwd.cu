// tc_bwd.cu -- chunkwise DDTS backward on the sm_100a tensor cores.
//
// The pages print no backward; this is the exact reverse mode of
//   S_t = diag(alpha_t) S_{t-1} + khat_t vhat_t^T,  o_t = S_t^T q_t,
// (alpha = exp(-g*tau), khat = g^tau * k, vhat = beta_hat * v; Rodimus*,
// digest.lyk-ai.com summary, "Method") organised by chunks of 64 tokens, last
// chunk first.  With b_t the inclusive running sum of log(alpha) in the chunk,
// m the per-channel reference of the forward (half the chunk's total, b_last / 2),
// Qt = q e^{b-m}, Kt = khat e^{m-b}, S_prev the state before the chunk (saved by
// the forward) and R = dL/dS at the end of the chunk (flowing backwards):
//
//   A  = mask_{s<=t}(Qt Kt^T)          B  = mask_{s<=t}(dO Vh^T)
//   dQ = B Kt + dO (diag(e^m) S_prev)^T          dq_t    = e^{b_t-m}  dQ_t
//   dK = B^T Qt + Vh (diag(e^{b_last-m}) R)^T    dkhat_s = e^{m-b_s}  dK_s
//   dV = A^T dO + Kt (diag(e^{b_last-m}) R)      dvhat_s = dV_s
//   R <- diag(e^{b_last}) R + diag(e^m) Qt^T dO  (becomes dL/dS_0 after chunk 0)
//
// and the decay gradient through the identity, exact for the closed form
// S_t = sum_s diag(e^{G_t-G_s}) khat_s vhat_s^T + diag(e^{G_t}) S_0:
//   d log(alpha_t) = sum_{u>=t} (q_u dq_u - khat_u dkhat_u)  [+ rowsum(dS_T o S_T)]
//   dk = alpha_hat dkhat,  dg = -tau dla + tau g^(tau-1) k dkhat,
//   dtau = -g dla + alpha_hat ln(g) k dkhat,  dv = beta dvhat,  dbeta = v dvhat.
//
// One CTA per (b,h) (d_k = 64, d_v = 64 or 128), 448 threads:
//   warps 0-3 epilogue (TMEM rows; R in fp32 registers), warps 4-11 gates
//   (operands before the MMAs, final gate gradients and the suffix scan after),
//   warp 12 TMA producer, warp 13 TMEM allocator + single-thread MMA issuer.
// A chunk whose log-decay span exceeds the range one reference can hold flags
// its head; those heads are recomputed afterwards by the exact CUDA-core
// backward (launched behind this kernel, it skips unflagged heads).
//
// Sequence segments (when the heads alone do not fill the GPU): each head's
// chunks are cut into P contiguous segments, one CTA each.  R maps affinely
// across a segment, R_start = diag(D) R_end + R_loc, so every segment but the
// first first computes R_loc alone (q, g, tau and dO only) and publishes
// (R_loc, log2 D); a segment then folds the maps of all later segments onto
// dS_T to obtain its R_end.  With G_t the running sum of log(alpha) from the
// segment start, R_loc = sum_t (q_t exp(G_t)) dO_t^T, every factor <= 1: the
// products of all its chunks accumulate into one tensor-memory sum (chunks
// taken first to last, which gives G_t as a running sum).  The decay-gradient carry
// into a segment, the suffix sum of (q dq - khat dkhat) over all later tokens
// plus rowsum(dS_T o S_T), equals rowsum(R_end o S_end) with S_end the state
// at the segment end (rescaling row i of q by e^eps and of khat and S_0 by
// e^-eps leaves o unchanged and scales S_T by e^-eps).  All CTAs of such a
// launch are resident together (cooperative launch); waits are bounded.
#include <cuda.h>

#include "launch.h"
#include "rdm_common.cuh"
#include "tc_common.cuh"

namespace rdm {
namespace {
using namespace tc;

constexpr int C = 64;
constexpr int DK = 64;
constexpr int kGateWarps = 8;  // one 8-channel group each
constexpr int kThreads = 32 * (4 + kGateWarps + 2);
constexpr int kEpiWarp0 = 0, kGateWarp0 = 4, kProdWarp = 4 + kGateWarps, kMmaWarp = 5 + kGateWarps;
constexpr int kBarEpi = 3;   // named barrier of the four epilogue warps
constexpr int kBarGate = 4;  // named barrier of the gate warps
constexpr int kStg = 68;
// row stride (floats) of the chunk-start state copied into shared memory: a
// 16-byte skew per row keeps the S_hat conversion free of bank conflicts
template <int DV>
constexpr int kSpStride = DV + 4;     // row stride (floats) of the dQ / dK staging tiles

template <int DV>
struct BCfg {
    static constexpr int VB = DV / 64;
    static constexpr int RAW = (4 + 3 * VB) * kBox;  // q k g tau | v beta dO
    static constexpr int OFF_V = 4 * kBox, OFF_B = (4 + VB) * kBox, OFF_DO = (4 + 2 * VB) * kBox;
    static constexpr int COL_A = 0, COL_B = 64, COL_DQ = 128, COL_DK = 192, COL_DV = 256,
                         COL_DR = 256 + DV;
    static constexpr int TMEM_COLS = 512;
};

template <int DV>
struct alignas(1024) BwdSmem {
    uint8_t raw[BCfg<DV>::RAW];
    // Vh and dO operands (no-swizzle layouts); once the second MMA group has
    // completed, the same bytes stage dv | dbeta for their TMA stores
    // (128B-swizzled, hence their 1024-byte aligned place after the raw tiles)
    uint8_t vh[C * DV * 2];    // [s][j], column groups 1024 B apart
    uint8_t dot[C * DV * 2];   // [t][j]
    uint8_t qt[8 * kQK];       // [t][i]
    uint8_t kt[8 * kQK];       // [s][i]
    uint8_t qtl[8 * kQK];      // bf16 remainders Qt - bf16(Qt), Kt - bf16(Kt): the
    uint8_t ktl[8 * kQK];      // pair products of dQ and dK reach ~16 mantissa bits
    // A, B and R_hat operands of the second MMA group; once that group has
    // completed, the same bytes hold the fp32 dQ / dK staging tiles; before the
    // first stage of the epilogue writes A, they hold the chunk-start state
    // S_prev (fp32) that the gate warps turn into S_hat
    union alignas(1024) {
        float sprev[DK * kSpStride<DV>];
        struct {
            uint8_t abf[C * C * 2];       // [t][s]
            uint8_t bmb[C * C * 2];       // [t][s]
            uint8_t rhat[DK * DV * 2];    // [i][j], e^{b_last-m} R
        } op;
        struct {
            float dqs[C][kStg], dks[C][kStg];
        } st;
    } u;
    uint8_t shat[DK * DV * 2];  // [i][j], e^m S_prev (written by the gate warps)
    float em[DK], cf[DK], gm[DK], fin[DK], carry[DK];
    float bdiag[C];  // B_tt = vhat_t . dO_t (the diagonal kept out of the dQ / dK MMAs)
    uint64_t raw_full, rawv_full, raw_empty, sp_full, ops_full, shat_full, ops_empty, g1_done, g2_ready,
        tm1_free, g2_done, tm2_free, post_ready, post_done, p1_done, vh_free;
    uint32_t tmem_base;
    int fail;
    int epi_fail;  // the epilogue's own exit decision (written before a role barrier)
};

// Segment exchange area (global): per (segment > 0, head) R_loc [DK][DV] and
// log2 of the decay product per channel; per (segment, head) a flag holding
// `tag` once those are written.
struct BwdSeg {
    int P;
    unsigned tag;
    float* st;
    float* ld;
    unsigned* flag;
};

struct BwdKernelArgs {
    CUtensorMap mq, mk, mg, mt, mv, mb, mdo;
    CUtensorMap mdq, mdk, mdg, mdt, mdv, mdb;  // gradient outputs (TMA stores)
    BwdParams p;
    int* flags;
    BwdSeg seg;
};

// Arrive `n` times at once on a CTA-local mbarrier.
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}

// [row][col] tile with 8-row groups 128 B apart and 8-column groups 1024 B
// apart (64 rows): K-major for (rows = M/N, K = cols), MN-major for (MN = cols,
// K = rows).
__device__ __forceinline__ uint32_t off_rc(int r, int c) {
    return (uint32_t)((r >> 3) * 128 + (c >> 3) * 1024 + (r & 7) * 16 + (c & 7) * 2);
}

// PRE: g, tau, beta arrive before their activations (gradients with respect to those)
template <int DV, bool PRE>
__global__ void __launch_bounds__(kThreads, 1) tc_bwd_kernel(const __grid_constant__ BwdKernelArgs A) {
    using K = BCfg<DV>;
    constexpr int VB = K::VB;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    BwdSmem<DV>& sm = *reinterpret_cast<BwdSmem<DV>*>(
        smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
    const BwdParams& p = A.p;
    const long long WL = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;  // bound of every wait
    const BwdSeg& sg = A.seg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.B * p.H;
    const int bh = blockIdx.x % BH, seg = blockIdx.x / BH;
    const int T = p.T, NC = (T + C - 1) / C;
    const int P = sg.P;
    const int cs0 = (int)((long long)seg * NC / P), cs1 = (int)((long long)(seg + 1) * NC / P);
    const int nseg = cs1 - cs0;
    const bool has_p1 = seg > 0;             // runs the R-only first pass
    const bool last_seg = seg == P - 1;      // its R_end is dS_T
    // chunk passes: the R-only pass over [cs0, cs1) first chunk first, then the
    // full pass last chunk first
    const int nL = (has_p1 ? 2 : 1) * nseg;
    auto pass_chunk = [&](int li) {
        return !has_p1 ? cs1 - 1 - li : li < nseg ? cs0 + li : cs1 - 1 - (li - nseg);
    };
    auto pass_p2 = [&](int li) { return !has_p1 || li >= nseg; };

    if (threadIdx.x == 0) {
        mbar_init(&sm.raw_full, 1);   // q, k, g, tau
        mbar_init(&sm.rawv_full, 1);  // v, beta, dO
        mbar_init(&sm.raw_empty, kGateWarps + 4);  // the epilogue reads v, beta, dO too
        mbar_init(&sm.sp_full, 1);
        mbar_init(&sm.ops_full, kGateWarps);
        mbar_init(&sm.shat_full, kGateWarps);
        mbar_init(&sm.ops_empty, 1);
        mbar_init(&sm.g1_done, 1);
        mbar_init(&sm.g2_ready, 4);
        mbar_init(&sm.tm1_free, 4);
        mbar_init(&sm.g2_done, 1);
        mbar_init(&sm.tm2_free, 4);
        mbar_init(&sm.post_ready, 4);
        mbar_init(&sm.post_done, kGateWarps);
        mbar_init(&sm.p1_done, kGateWarps);
        mbar_init(&sm.vh_free, 1);
        sm.epi_fail = 0;
        sm.fail = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < DK) {
        sm.fin[threadIdx.x] = 0.0f;
        sm.carry[threadIdx.x] = 0.0f;
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, K::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_tmap(&A.mq); prefetch_tmap(&A.mk); prefetch_tmap(&A.mg); prefetch_tmap(&A.mt);
        prefetch_tmap(&A.mv); prefetch_tmap(&A.mb); prefetch_tmap(&A.mdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* fail = &sm.fail;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0, issued_sp = 0;
            for (int li = 0; li < nL; ++li) {
                const int c = pass_chunk(li);
                const bool p2 = pass_p2(li);
                if (li > 0 && !mbar_wait(&sm.raw_empty, (li - 1) & 1, fail, WL)) break;
                // the R-only pass reads q, g, tau and dO
                // the key side first (the gate warps start with its scan), then the
                // value side on its own barrier
                mbar_expect_tx(&sm.raw_full, (p2 ? 4 : 3) * kBox);
                tma_load_3d(sm.raw + 2 * kBox, &A.mg, &sm.raw_full, 0, c * C, bh);
                tma_load_3d(sm.raw + 3 * kBox, &A.mt, &sm.raw_full, 0, c * C, bh);
                tma_load_3d(sm.raw + 0 * kBox, &A.mq, &sm.raw_full, 0, c * C, bh);
                if (p2) tma_load_3d(sm.raw + 1 * kBox, &A.mk, &sm.raw_full, 0, c * C, bh);
                // the R-only pass reads dO only
                mbar_expect_tx(&sm.rawv_full, (p2 ? 3 : 1) * VB * kBox);
                for (int vb = 0; vb < VB; ++vb) {
                    if (p2) {
                        tma_load_3d(sm.raw + K::OFF_V + vb * kBox, &A.mv, &sm.rawv_full, 64 * vb, c * C, bh);
                        tma_load_3d(sm.raw + K::OFF_B + vb * kBox, &A.mb, &sm.rawv_full, 64 * vb, c * C, bh);
                    }
                    tma_load_3d(sm.raw + K::OFF_DO + vb * kBox, &A.mdo, &sm.rawv_full, 64 * vb, c * C, bh);
                }
                ++issued;
                // the next pass's tiles (and chunk-start state) into L2 while this one runs
                if (li + 1 < nL) {
                    const int cn = pass_chunk(li + 1);
                    const bool pn = pass_p2(li + 1);
                    tma_prefetch_3d(&A.mq, 0, cn * C, bh);
                    if (pn) tma_prefetch_3d(&A.mk, 0, cn * C, bh);
                    tma_prefetch_3d(&A.mg, 0, cn * C, bh);
                    tma_prefetch_3d(&A.mt, 0, cn * C, bh);
                    for (int vb = 0; vb < VB; ++vb) {
                        if (pn) {
                            tma_prefetch_3d(&A.mv, 64 * vb, cn * C, bh);
                            tma_prefetch_3d(&A.mb, 64 * vb, cn * C, bh);
                        }
                        tma_prefetch_3d(&A.mdo, 64 * vb, cn * C, bh);
                    }
                    if (pn) bulk_prefetch_l2(p.saved + ((size_t)bh * NC + cn) * DK * DV, DK * DV * 4);
                }
                if (p2) {
                    // chunk-start state, row by row into the skewed layout (the union
                    // is free: the previous full pass has finished its last stage)
                    const float* Sp = p.saved + ((size_t)bh * NC + c) * DK * DV;
                    mbar_expect_tx(&sm.sp_full, DK * DV * 4);
                    for (int i = 0; i < DK; ++i)
                        bulk_load(sm.u.sprev + i * kSpStride<DV>, Sp + (size_t)i * DV, DV * 4, &sm.sp_full);
                    ++issued_sp;
                }
            }
            if (issued > 0) {
                drain_wait(&sm.raw_full, (issued - 1) & 1);
                drain_wait(&sm.rawv_full, (issued - 1) & 1);
            }
            if (issued_sp > 0) drain_wait(&sm.sp_full, (issued_sp - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q = smem_u32(sm.qt), k = smem_u32(sm.kt), v = smem_u32(sm.vh);
            const uint32_t d = smem_u32(sm.dot), a = smem_u32(sm.u.op.abf), bm = smem_u32(sm.u.op.bmb);
            const uint32_t sh = smem_u32(sm.shat), rh = smem_u32(sm.u.op.rhat);
            const uint32_t ql = smem_u32(sm.qtl), kl = smem_u32(sm.ktl);
            constexpr uint32_t id_a = idesc_bf16(64, 64, 0, 0);    // A = Qt Kt^T, B = dO Vh^T
            constexpr uint32_t id_r = idesc_bf16(DK, DV, 1, 1);    // Qt^T dO, Kt^T Vh
            constexpr uint32_t id_q1 = idesc_bf16(64, DK, 0, 1);   // B Kt
            constexpr uint32_t id_q2 = idesc_bf16(64, DK, 0, 0);   // dO S_hat^T
            constexpr uint32_t id_k1 = idesc_bf16(64, DK, 1, 1);   // B^T Qt
            constexpr uint32_t id_k2 = idesc_bf16(64, DK, 0, 0);   // Vh R_hat^T
            constexpr uint32_t id_v1 = idesc_bf16(64, DV, 1, 1);   // A^T dO
            constexpr uint32_t id_v2 = idesc_bf16(64, DV, 0, 1);   // Kt R_hat
            int n1 = 0, n2 = 0;
            for (int li = 0; li < nL; ++li) {
                const bool p2 = pass_p2(li);
                const int i2 = n2;  // index among full passes
                if (!mbar_wait(&sm.ops_full, li & 1, fail, WL)) break;
                // group-1 accumulators released by the epilogue: after the R-only
                // pass, and after each full pass (tm1_free completes once for each)
                const int ntf = i2 + (has_p1 ? 1 : 0);
                if (p2 && ntf > 0 && !mbar_wait(&sm.tm1_free, (ntf - 1) & 1, fail, WL)) break;
                tc_fence_after();
                if (!p2) {
                    // R-only pass: R_loc += Qt^T dO over all its chunks
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        mma_bf16(tmem + K::COL_DR, sdesc(q + ks * 256, 128, kQK),
                                 sdesc(d + ks * 256, 128, 1024), id_r, ks > 0 || li > 0);
                    if (li == nseg - 1) {
                        mma_commit(&sm.g1_done);
                        ++n1;
                    }
                    mma_commit(&sm.ops_empty);
                    continue;
                }
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    mma_bf16(tmem + K::COL_A, sdesc(q + ks * 2 * kQK, kQK, 128),
                             sdesc(k + ks * 2 * kQK, kQK, 128), id_a, ks > 0);
#pragma unroll
                for (int ks = 0; ks < DV / 16; ++ks)
                    mma_bf16(tmem + K::COL_B, sdesc(d + ks * 2048, 1024, 128),
                             sdesc(v + ks * 2048, 1024, 128), id_a, ks > 0);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DR, sdesc(q + ks * 256, 128, kQK),
                             sdesc(d + ks * 256, 128, 1024), id_r, ks > 0);
                // and with Qt's bf16 remainder: R (hence dS_0 and the segment carries)
                // to ~16 mantissa bits
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DR, sdesc(ql + ks * 256, 128, kQK),
                             sdesc(d + ks * 256, 128, 1024), id_r, 1);
                if (i2 == 0 && last_seg && p.dST) {
                    // Kt^T Vh of the last chunk, for S_T (only the final-state gradient needs it)
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        mma_bf16(tmem + K::COL_DV, sdesc(k + ks * 256, 128, kQK),
                                 sdesc(v + ks * 256, 128, 1024), id_r, ks > 0);
                }
                mma_commit(&sm.g1_done);
                ++n1;
                if (!mbar_wait(&sm.g2_ready, i2 & 1, fail, WL)) break;
                if (!mbar_wait(&sm.shat_full, i2 & 1, fail, WL)) break;
                if (i2 > 0 && !mbar_wait(&sm.tm2_free, (i2 - 1) & 1, fail, WL)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DQ, sdesc(bm + ks * 2048, 1024, 128),
                             sdesc(k + ks * 256, 128, kQK), id_q1, ks > 0);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DQ, sdesc(bm + ks * 2048, 1024, 128),
                             sdesc(kl + ks * 256, 128, kQK), id_q1, 1);
#pragma unroll
                for (int ks = 0; ks < DV / 16; ++ks)
                    mma_bf16(tmem + K::COL_DQ, sdesc(d + ks * 2048, 1024, 128),
                             sdesc(sh + ks * 2048, 1024, 128), id_q2, 1);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DK, sdesc(bm + ks * 256, 128, 1024),
                             sdesc(q + ks * 256, 128, kQK), id_k1, ks > 0);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DK, sdesc(bm + ks * 256, 128, 1024),
                             sdesc(ql + ks * 256, 128, kQK), id_k1, 1);
#pragma unroll
                for (int ks = 0; ks < DV / 16; ++ks)
                    mma_bf16(tmem + K::COL_DK, sdesc(v + ks * 2048, 1024, 128),
                             sdesc(rh + ks * 2048, 1024, 128), id_k2, 1);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + K::COL_DV, sdesc(a + ks * 256, 128, 1024),
                             sdesc(d + ks * 256, 128, 1024), id_v1, ks > 0);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    mma_bf16(tmem + K::COL_DV, sdesc(k + ks * 2 * kQK, kQK, 128),
                             sdesc(rh + ks * 256, 128, 1024), id_v2, 1);
                mma_commit(&sm.g2_done);
                mma_commit(&sm.ops_empty);
                ++n2;
            }
            if (n1 > 0) drain_wait(&sm.g1_done, (n1 - 1) & 1);
            if (n2 > 0) drain_wait(&sm.g2_done, (n2 - 1) & 1);
        }
        __syncwarp();
    } else if (warp >= kGateWarp0) {
        // ------------------------------------------------------------ gates
        // warp gw owns channel group gw (8 channels) for all 64 tokens; lane ->
        // segment of SEGT tokens.  Prefix (running log-decay) and suffix (decay
        // gradient) scans are in-thread plus shuffles: no data crosses warps.
        constexpr int G = DK / 8, GW = G / kGateWarps, NSW = 32 / GW, SEGT = C / NSW;
        constexpr int VG = DV / 8, TPG = 32 * kGateWarps / VG, VIT = C / TPG;
        const int gw = warp - kGateWarp0, gt = gw * 32 + lane;
        const int cgl = lane % GW, seg = lane / GW;
        const int cg = gw * GW + cgl;
        const int tb = seg * SEGT;
        const uint32_t full = 0xffffffffu;
        const uint8_t* raw = sm.raw;
        int i2 = 0;  // full passes done
        float gh2[8];  // R-only pass: log2 decay from the segment start to this chunk
#pragma unroll
        for (int e = 0; e < 8; ++e) gh2[e] = 0.0f;
        for (int li = 0; li < nL; ++li) {
            const int c = pass_chunk(li);
            const bool p2 = pass_p2(li);
            if (!mbar_wait_own(&sm.raw_full, li & 1, fail, WL)) break;
            const int nval = min(C, T - c * C);
            // ---- pre: running log-decay, reference, operands
            float b[SEGT][8], mL[8], blL[8];
#pragma unroll
            for (int u = 0; u < SEGT; ++u) {
                float g8[8], t8[8];
                unpack8(*reinterpret_cast<const uint4*>(raw + 2 * kBox + off_raw(tb + u, cg)), g8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 3 * kBox + off_raw(tb + u, cg)), t8);
                if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float la = (tb + u < nval) ? log_alpha(g8[e], t8[e]) : 0.0f;
                    b[u][e] = u == 0 ? la : b[u - 1][e] + la;
                }
            }
            {
                const int tl = nval - 1;
                const int lsrc = cgl + GW * (tl / SEGT), usrc = tl % SEGT;
                float span = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float tot = b[SEGT - 1][e];
                    float x = tot;
#pragma unroll
                    for (int d = GW; d < 32; d <<= 1) {
                        const float y = __shfl_up_sync(full, x, d);
                        if (lane >= d) x += y;
                    }
                    float mine = 0.0f;
#pragma unroll
                    for (int u = 0; u < SEGT; ++u) {
                        b[u][e] += x - tot;
                        if (u == usrc) mine = b[u][e];
                    }
                    // reference m = half the chunk's total log decay: b runs over
                    // [b_last, 0], so every factor stays inside exp(+-|b_last|/2)
                    const float bl = __shfl_sync(full, mine, lsrc);
                    mL[e] = 0.5f * bl * kLog2e;
                    blL[e] = bl * kLog2e;
                    span = fmaxf(span, -bl);
                }
                // too wide for one reference: the exact path recomputes this head
                // (the R-only pass needs no reference)
                if (p2 && __any_sync(full, !(span <= kSpanMax)) && lane == 0) A.flags[bh] = 1;
            }
            // operand slot free: tensor core done with it (ops_empty) and, for a full
            // pass, the epilogue done with the constants (tm1_free, once after the
            // R-only pass and once per full pass; it consumes em / cf / gm in its
            // first stage)
            if (li > 0 && !mbar_wait_own(&sm.ops_empty, (li - 1) & 1, fail, WL)) break;
            if (p2) {
                const int ntf = i2 + (has_p1 ? 1 : 0);
                if (ntf > 0 && !mbar_wait_own(&sm.tm1_free, (ntf - 1) & 1, fail, WL)) break;
            }
            if (!p2) {
                // R-only pass: Qt = q exp(G_t) relative to the segment start (gh2 the
                // decay of the earlier chunks, log2; every factor <= 1), and dO
#pragma unroll
                for (int u = 0; u < SEGT; ++u) {
                    const int t = tb + u;
                    float q8[8], oq[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 0 * kBox + off_raw(t, cg)), q8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) oq[e] = q8[e] * ex2_fast(fmaf(b[u][e], kLog2e, gh2[e]));
                    *reinterpret_cast<uint4*>(sm.qt + off_qk(t, cg * 8)) = pack8(oq);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) gh2[e] += blL[e];
                const bool p1last = li == nseg - 1;
                // log2 of the segment's decay product, for the epilogue
                if (p1last && tb == 0) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) sm.gm[cg * 8 + e] = gh2[e];
                }
                if (!mbar_wait_own(&sm.rawv_full, li & 1, fail, WL)) break;
#pragma unroll
                for (int iv = 0; iv < VIT; ++iv) {
                    const int jg = gt / TPG, t = (gt % TPG) + TPG * iv;
                    *reinterpret_cast<uint4*>(sm.dot + off_rc(t, jg * 8)) =
                        *reinterpret_cast<const uint4*>(raw + K::OFF_DO + off_raw(t, jg));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sm.ops_full);
                    // the epilogue reads no raw tile in this pass: warp 0 arrives
                    // for its four warps as well
                    if (gw == 0) mbar_arrive_n(&sm.raw_empty, 5);
                    else mbar_arrive(&sm.raw_empty);
                    if (p1last) mbar_arrive(&sm.p1_done);
                }
                continue;
            }
#pragma unroll
            for (int u = 0; u < SEGT; ++u) {
                const int t = tb + u;
                float q8[8], k8[8], g8[8], t8[8], oq[8], ok[8];
                unpack8(*reinterpret_cast<const uint4*>(raw + 0 * kBox + off_raw(t, cg)), q8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 1 * kBox + off_raw(t, cg)), k8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 2 * kBox + off_raw(t, cg)), g8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 3 * kBox + off_raw(t, cg)), t8);
                if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float dd = fmaf(b[u][e], kLog2e, -mL[e]);
                    const float lah = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                    oq[e] = q8[e] * ex2_fast(dd);
                    ok[e] = k8[e] * ex2_fast(lah - dd);
                }
                const uint4 hq = pack8(oq), hk = pack8(ok);
                float fq[8], fk[8];
                unpack8(hq, fq);
                unpack8(hk, fk);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    oq[e] -= fq[e];
                    ok[e] -= fk[e];
                }
                *reinterpret_cast<uint4*>(sm.qt + off_qk(t, cg * 8)) = hq;
                *reinterpret_cast<uint4*>(sm.kt + off_qk(t, cg * 8)) = hk;
                *reinterpret_cast<uint4*>(sm.qtl + off_qk(t, cg * 8)) = pack8(oq);
                *reinterpret_cast<uint4*>(sm.ktl + off_qk(t, cg * 8)) = pack8(ok);
            }
            if (tb == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sm.em[cg * 8 + e] = ex2_fast(mL[e]);
                    sm.cf[cg * 8 + e] = ex2_fast(blL[e] - mL[e]);
                    sm.gm[cg * 8 + e] = ex2_fast(blL[e]);
                }
            }
            // Vh and dO operand buffers: the epilogue's dv / dbeta stores of the
            // previous chunk have read them
            if (i2 > 0 && !mbar_wait_own(&sm.vh_free, (i2 - 1) & 1, fail, WL)) break;
            if (!mbar_wait_own(&sm.rawv_full, li & 1, fail, WL)) break;
#pragma unroll
            for (int iv = 0; iv < VIT; ++iv) {
                const int jg = gt / TPG, t = (gt % TPG) + TPG * iv;
                float v8[8], b8[8], o8[8];
                unpack8(*reinterpret_cast<const uint4*>(raw + K::OFF_V + off_raw(t, jg)), v8);
                unpack8(*reinterpret_cast<const uint4*>(raw + K::OFF_B + off_raw(t, jg)), b8);
                if constexpr (PRE) activate_beta8(b8);
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = v8[e] * b8[e];
                *reinterpret_cast<uint4*>(sm.vh + off_rc(t, jg * 8)) = pack8(o8);
                *reinterpret_cast<uint4*>(sm.dot + off_rc(t, jg * 8)) =
                    *reinterpret_cast<const uint4*>(raw + K::OFF_DO + off_raw(t, jg));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.ops_full);
            // S_hat = diag(e^m) S_prev for this warp's rows (channels), while the
            // first MMA group runs
            if (!mbar_wait_own(&sm.sp_full, i2 & 1, fail, WL)) break;
#pragma unroll
            for (int gi = 0; gi < GW; ++gi) {
                const int i = (gw * GW + gi) * 8 + (lane >> 2);
                const float* Sp = sm.u.sprev + i * kSpStride<DV>;
                constexpr int CPT = DV / 4;  // 8 rows x DV columns over 32 lanes
                const int c0 = (lane & 3) * CPT;
                const float emr = sm.em[i];
#pragma unroll
                for (int j8 = 0; j8 < CPT / 8; ++j8) {
                    const float4 s0 = *reinterpret_cast<const float4*>(Sp + c0 + 8 * j8);
                    const float4 s1 = *reinterpret_cast<const float4*>(Sp + c0 + 8 * j8 + 4);
                    const float xs[8] = {s0.x * emr, s0.y * emr, s0.z * emr, s0.w * emr,
                                         s1.x * emr, s1.y * emr, s1.z * emr, s1.w * emr};
                    *reinterpret_cast<uint4*>(sm.shat + off_rc(i, c0 + 8 * j8)) = pack8(xs);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.shat_full);

            // ---- post: final gate gradients once dQ, dK of this chunk are staged
            if (!mbar_wait_own(&sm.post_ready, i2 & 1, fail, WL)) break;
            uint8_t* gst = sm.qt;  // 4 x 8 KB over qt | kt | qtl | ktl
            float dG[SEGT][8], dkh[SEGT][8];
#pragma unroll
            for (int u = 0; u < SEGT; ++u) {
                const int t = tb + u;
                float q8[8], k8[8], g8[8], t8[8], dqo[8];
                unpack8(*reinterpret_cast<const uint4*>(raw + 0 * kBox + off_raw(t, cg)), q8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 1 * kBox + off_raw(t, cg)), k8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 2 * kBox + off_raw(t, cg)), g8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 3 * kBox + off_raw(t, cg)), t8);
                if constexpr (PRE) activate_gates8(g8, t8);
                const float4* dq4 = reinterpret_cast<const float4*>(&sm.u.st.dqs[t][cg * 8]);
                const float4* dk4 = reinterpret_cast<const float4*>(&sm.u.st.dks[t][cg * 8]);
                const float4 qa = dq4[0], qb = dq4[1], ka = dk4[0], kb4 = dk4[1];
                const float dQv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
                const float dKv[8] = {ka.x, ka.y, ka.z, ka.w, kb4.x, kb4.y, kb4.z, kb4.w};
                const float bd = sm.bdiag[t];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float dd = fmaf(b[u][e], kLog2e, -mL[e]);
                    const float lah = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                    const float kh = ex2_fast(lah) * k8[e];
                    const float dq_off = ex2_fast(dd) * dQv[e];    // pairs s < t
                    const float dk_off = ex2_fast(-dd) * dKv[e];   // pairs t > s
                    dG[u][e] = q8[e] * dq_off - kh * dk_off;        // the s = t pair cancels
                    dqo[e] = dq_off + kh * bd;
                    dkh[u][e] = dk_off + q8[e] * bd;
                }
                // staged in the (now idle) Qt / Kt operand buffers, stored by TMA below
                *reinterpret_cast<uint4*>(gst + 0 * kBox + off_raw(t, cg)) = pack8(dqo);
            }
            // d log(alpha) = suffix sum of dG: in the segment, over later segments of
            // this warp (= later tokens of the chunk), over later chunks (carry)
#pragma unroll
            for (int u = SEGT - 2; u >= 0; --u)
#pragma unroll
                for (int e = 0; e < 8; ++e) dG[u][e] += dG[u + 1][e];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float tot = dG[0][e];
                float x = tot;
#pragma unroll
                for (int d = GW; d < 32; d <<= 1) {
                    const float y = __shfl_down_sync(full, x, d);
                    if (lane + d < 32) x += y;
                }
                const float off = (x - tot) + sm.carry[cg * 8 + e] +
                                  (i2 == 0 && last_seg ? sm.fin[cg * 8 + e] : 0.0f);
#pragma unroll
                for (int u = 0; u < SEGT; ++u) dG[u][e] += off;
            }
#pragma unroll
            for (int u = 0; u < SEGT; ++u) {
                const int t = tb + u;
                float k8[8], g8[8], t8[8], odk[8], odg[8], odt[8];
                unpack8(*reinterpret_cast<const uint4*>(raw + 1 * kBox + off_raw(t, cg)), k8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 2 * kBox + off_raw(t, cg)), g8);
                unpack8(*reinterpret_cast<const uint4*>(raw + 3 * kBox + off_raw(t, cg)), t8);
                // chain factors to the pre-activations: softplus' = sigmoid, sigmoid' = s (1 - s)
                float cgf[8], ctf[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cgf[e] = 1.0f;
                    ctf[e] = 1.0f;
                    if constexpr (PRE) {
                        cgf[e] = sigmoid_fast(g8[e]);
                        g8[e] = softplus_fast(g8[e]);
                        t8[e] = sigmoid_fast(t8[e]);
                        ctf[e] = t8[e] * (1.0f - t8[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float gg = g8[e], ta = t8[e];
                    const float l2g = lg2_fast(gg);
                    const float ah = ta == 0.0f ? 1.0f : ex2_fast(ta * l2g);
                    const float dah = k8[e] * dkh[u][e];
                    const float dah_dg = ta == 0.0f ? 0.0f : ta * ex2_fast((ta - 1.0f) * l2g);
                    const float dah_dt = ah == 0.0f ? 0.0f : ah * l2g * kLn2;
                    odk[e] = ah * dkh[u][e];
                    odg[e] = cgf[e] * (-ta * dG[u][e] + dah_dg * dah);
                    odt[e] = ctf[e] * (-gg * dG[u][e] + dah_dt * dah);
                }
                *reinterpret_cast<uint4*>(gst + 1 * kBox + off_raw(t, cg)) = pack8(odk);
                *reinterpret_cast<uint4*>(gst + 2 * kBox + off_raw(t, cg)) = pack8(odg);
                *reinterpret_cast<uint4*>(gst + 3 * kBox + off_raw(t, cg)) = pack8(odt);
            }
            // this warp's last read of the raw tiles and of the dQ / dK staging (the
            // epilogue read its raw rows before it handed over the staging): the
            // producer may load the next chunk while the gradients are stored
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.raw_empty);
            // dq, dk, dg, dtau of the chunk: one TMA store each (rows past T are
            // clipped); the staging bytes are read before the next operand stage
            fence_proxy_async_smem();
            named_bar(kBarGate, 32 * kGateWarps);
            if (gt == 0) {
                tma_store_3d(&A.mdq, gst + 0 * kBox, 0, c * C, bh);
                tma_store_3d(&A.mdk, gst + 1 * kBox, 0, c * C, bh);
                tma_store_3d(&A.mdg, gst + 2 * kBox, 0, c * C, bh);
                tma_store_3d(&A.mdt, gst + 3 * kBox, 0, c * C, bh);
                bulk_commit();
                bulk_wait_read_all();
            }
            named_bar(kBarGate, 32 * kGateWarps);
            __syncwarp();  // every lane has read the old carry
            if (tb == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) sm.carry[cg * 8 + e] = dG[0][e];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.post_done);
            ++i2;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // M = 64 accumulators sit in TMEM lanes 0-15 of each sub-partition; the
        // split load hands row r = 16 ew + (lane & 15) to two threads, lane >> 4
        // selecting which half of the columns each one holds.
        constexpr int HV = DV / 2;  // state columns per thread
        const int ew = warp - kEpiWarp0;
        const int hf = lane >> 4;
        const int r = 16 * ew + (lane & 15);
        const uint32_t lb = (uint32_t)(32 * ew) << 16;
        float R[HV];  // R[r][hf*HV .. hf*HV + HV)
        auto load_dst = [&]() {
#pragma unroll
            for (int j = 0; j < HV; ++j)
                R[j] = p.dST ? p.dST[((size_t)bh * DK + r) * DV + hf * HV + j] : 0.0f;
        };
        // A segment's map in the workspace is kept in the epilogue's register
        // order (float4 k of thread et at k * 128 + et), so that every warp
        // instruction reads or writes 512 contiguous bytes.
        auto seg_map_ptr = [&](size_t u) {
            return reinterpret_cast<float4*>(sg.st) + u * (DK * DV / 4) + (threadIdx.x - 32 * kEpiWarp0);
        };
        // R at the end of this segment: dS_T carried through the maps of all later
        // segments, R <- diag(D_s) R + R_loc_s; then the decay-gradient carry into
        // the segment, rowsum(R o S) with S the saved state at the segment end
        auto fold_later = [&]() -> bool {
            if (threadIdx.x == 0) {
                const long long t0 = clock64();
                for (int s2 = P - 1; s2 > seg && !*fail; --s2)
                    while (ld_acquire_gpu(&sg.flag[s2 * BH + bh]) != sg.tag)
                        if (clock64() - t0 > WL) {
                            *fail = 1;
                            sm.epi_fail = 1;
                            break;
                        }
            }
            named_bar(kBarEpi, 128);
            if (sm.epi_fail) return false;  // written by thread 0 before the barrier
            load_dst();
            for (int s2 = P - 1; s2 > seg; --s2) {
                const size_t u = (size_t)s2 * BH + bh;
                const float d = ex2_fast(__ldcg(&sg.ld[u * DK + r]));
                const float4* src = seg_map_ptr(u);
#pragma unroll
                for (int j4 = 0; j4 < HV / 4; ++j4) {
                    const float4 x = __ldcg(src + j4 * 128);
                    R[4 * j4] = fmaf(d, R[4 * j4], x.x);
                    R[4 * j4 + 1] = fmaf(d, R[4 * j4 + 1], x.y);
                    R[4 * j4 + 2] = fmaf(d, R[4 * j4 + 2], x.z);
                    R[4 * j4 + 3] = fmaf(d, R[4 * j4 + 3], x.w);
                }
            }
            if (!last_seg) {
                const float* Se = p.saved + (((size_t)bh * NC + cs1) * DK + r) * DV + hf * HV;
                float f = 0.0f;
#pragma unroll
                for (int j = 0; j < HV; ++j) f = fmaf(R[j], Se[j], f);
                f += __shfl_xor_sync(0xffffffffu, f, 16);
                if (hf == 0) sm.carry[r] = f;
            }
            return true;
        };
        // publish this segment's map (R_loc in R, log2 D in ld2)
        auto publish_segment = [&](float ld2) -> bool {
            const size_t u = (size_t)seg * BH + bh;
            float4* dst = seg_map_ptr(u);
#pragma unroll
            for (int j4 = 0; j4 < HV / 4; ++j4)
                dst[j4 * 128] = make_float4(R[4 * j4], R[4 * j4 + 1], R[4 * j4 + 2], R[4 * j4 + 3]);
            if (hf == 0) sg.ld[u * DK + r] = ld2;
            __threadfence();
            named_bar(kBarEpi, 128);
            if (threadIdx.x == 0 && !p.withhold_flags) st_release_gpu(&sg.flag[u], sg.tag);
            return true;
        };
        bool ok_run = true;
        if (P == 1) {
            load_dst();
        } else if (has_p1) {
#pragma unroll
            for (int j = 0; j < HV; ++j) R[j] = 0.0f;
        } else {
            ok_run = fold_later();
        }
        int i2 = 0;  // full passes done
        if (ok_run && has_p1) {
            // R-only pass: R_loc is the accumulated group-1 sum once its last
            // chunk's products are done; log2 D comes from the gate warps
            ok_run = mbar_wait_own(&sm.p1_done, 0, fail, WL) &&
                     mbar_wait_own(&sm.g1_done, 0, fail, WL);
            if (ok_run) {
                tc_fence_after();
                const float ld2 = sm.gm[r];
#pragma unroll
                for (int qd = 0; qd < HV / 32; ++qd) {
                    tmem_ld32_split<HV>(tmem + lb + K::COL_DR + 32 * qd, R + 32 * qd);
                    tmem_ld_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tm1_free);
                ok_run = publish_segment(ld2) && fold_later();
            }
        }
        for (int li = has_p1 ? nseg : 0; ok_run && li < nL; ++li) {
            const int c = pass_chunk(li);
            if (!mbar_wait_own(&sm.ops_full, li & 1, fail, WL)) break;
            if (!mbar_wait_own(&sm.g1_done, (i2 + (has_p1 ? 1 : 0)) & 1, fail, WL)) break;
            tc_fence_after();
            // the gate warps have read S_prev out of the union (and staged S_hat)
            if (!mbar_wait_own(&sm.shat_full, i2 & 1, fail, WL)) break;
            // A and B -> causal mask -> bf16 operands (row t = r, columns s = 32 hf + e)
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                float v[32];
                tmem_ld32_split<32>(tmem + lb + (which == 0 ? K::COL_A : K::COL_B), v);
                tmem_ld_wait();
                uint8_t* dst = which == 0 ? sm.u.op.abf : sm.u.op.bmb;
                // A keeps s <= t.  B keeps s < t: its diagonal contributes the same
                // product to q.dq and to khat.dkhat, which cancel exactly in the
                // decay gradient, so it is added back in fp32 after the MMAs
                // instead of passing through two differently rounded operands.
                if (which == 1 && (r >> 5) == hf) {
                    float dg = 0.0f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) dg = (32 * hf + e == r) ? v[e] : dg;
                    sm.bdiag[r] = dg;
                }
                const int lim = (which == 0 ? r : r - 1) - 32 * hf;
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = (e <= lim) ? v[e] : 0.0f;
#pragma unroll
                for (int sg = 0; sg < 4; ++sg)
                    *reinterpret_cast<uint4*>(dst + off_rc(r, 32 * hf + 8 * sg)) = pack8(v + 8 * sg);
            }
            const float emv = sm.em[r], cfv = sm.cf[r], gmv = sm.gm[r];
            if (i2 == 0 && last_seg && p.dST) {
                // final-state term rowsum(dS_T o S_T) with S_T = diag(gm) S_prev + diag(cf) Kt^T Vh
                const float* Sprev = p.saved + (((size_t)bh * NC + c) * DK + r) * DV + hf * HV;
                float f = 0.0f;
#pragma unroll
                for (int qd = 0; qd < HV / 32; ++qd) {
                    float v[32];
                    tmem_ld32_split<HV>(tmem + lb + K::COL_DV + 32 * qd, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * qd + e;
                        f = fmaf(R[j], fmaf(gmv, Sprev[j], cfv * v[e]), f);  // R = dS_T here
                    }
                }
                f += __shfl_xor_sync(0xffffffffu, f, 16);
                if (hf == 0) sm.fin[r] = f;
            }
            // R_hat = diag(cf) R  (S_hat is written by the gate warps)
#pragma unroll
            for (int jg = 0; jg < HV / 8; ++jg) {
                float xr[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) xr[e] = R[8 * jg + e] * cfv;
                *reinterpret_cast<uint4*>(sm.u.op.rhat + off_rc(r, hf * HV + 8 * jg)) = pack8(xr);
            }
            // R <- diag(e^{b_last}) R + diag(e^m) Qt^T dO
#pragma unroll
            for (int qd = 0; qd < HV / 32; ++qd) {
                float v[32];
                tmem_ld32_split<HV>(tmem + lb + K::COL_DR + 32 * qd, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) R[32 * qd + e] = fmaf(gmv, R[32 * qd + e], emv * v[e]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.g2_ready);
                mbar_arrive(&sm.tm1_free);
            }
            if (!mbar_wait_own(&sm.g2_done, i2 & 1, fail, WL)) break;
            tc_fence_after();
            // dQ, dK -> fp32 staging for the gate warps first (the union: the
            // previous chunk's gate stage has read its staging), so that their final
            // stage runs beside the dv / dbeta stage below
            if (i2 > 0 && !mbar_wait_own(&sm.post_done, (i2 - 1) & 1, fail, WL)) break;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                float v[32];
                tmem_ld32_split<32>(tmem + lb + (which == 0 ? K::COL_DQ : K::COL_DK), v);
                tmem_ld_wait();
                float4* dst = reinterpret_cast<float4*>(which == 0 ? &sm.u.st.dqs[r][32 * hf] : &sm.u.st.dks[r][32 * hf]);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    dst[e4] = make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.post_ready);
            // dV -> dv = beta dvhat, dbeta = v dvhat (row s = r), staged in the Vh |
            // dO operand buffers (idle once the second group has completed) and
            // written by TMA stores
            {
#pragma unroll 1
                for (int qd = 0; qd < HV / 32; ++qd) {
                    float v[32];
                    tmem_ld32_split<HV>(tmem + lb + K::COL_DV + 32 * qd, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int h4 = 0; h4 < 4; ++h4) {
                        const int jg = (hf * HV + 32 * qd) / 8 + h4;
                        float v8[8], b8[8], ov[8], ob[8];
                        unpack8(*reinterpret_cast<const uint4*>(sm.raw + K::OFF_V + off_raw(r, jg)), v8);
                        unpack8(*reinterpret_cast<const uint4*>(sm.raw + K::OFF_B + off_raw(r, jg)), b8);
                        float cb[8];  // chain factor to the pre-activation of beta_hat
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            cb[e] = 1.0f;
                            if constexpr (PRE) {
                                b8[e] = sigmoid_tanh(b8[e]);
                                cb[e] = b8[e] * (1.0f - b8[e]);
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            ov[e] = b8[e] * v[8 * h4 + e];
                            ob[e] = cb[e] * v8[e] * v[8 * h4 + e];
                        }
                        if (p.dfeed != nullptr) {  // feedthrough: dv_t += d (.) dO_t
                            float do8[8];
                            unpack8(*reinterpret_cast<const uint4*>(sm.raw + K::OFF_DO + off_raw(r, jg)), do8);
                            const float4* dr = reinterpret_cast<const float4*>(p.dfeed + (size_t)(bh % p.H) * DV + 8 * jg);
                            const float4 d0 = __ldg(dr), d1 = __ldg(dr + 1);
                            const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                            for (int e = 0; e < 8; ++e) ov[e] = fmaf(dd[e], do8[e], ov[e]);
                        }
                        *reinterpret_cast<uint4*>(sm.vh + off_raw(r, jg)) = pack8(ov);
                        *reinterpret_cast<uint4*>(sm.dot + off_raw(r, jg)) = pack8(ob);
                    }
                }
                // this warp's last read of the raw tiles (v, beta, dO) and of TMEM
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sm.raw_empty);
                    mbar_arrive(&sm.tm2_free);
                }
                fence_proxy_async_smem();
                named_bar(kBarEpi, 128);
                if (threadIdx.x == 0) {
#pragma unroll
                    for (int vb = 0; vb < VB; ++vb) {
                        tma_store_3d(&A.mdv, sm.vh + vb * kBox, 64 * vb, c * C, bh);
                        tma_store_3d(&A.mdb, sm.dot + vb * kBox, 64 * vb, c * C, bh);
                    }
                    bulk_commit();
                    bulk_wait_read_all();  // the gate warps write the next chunk's operands there
                    mbar_arrive(&sm.vh_free);
                }
            }
            ++i2;
        }
        if (!*fail && p.dS0 && seg == 0) {
            float4* dst = reinterpret_cast<float4*>(p.dS0 + ((size_t)bh * DK + r) * DV + hf * HV);
#pragma unroll
            for (int j4 = 0; j4 < HV / 4; ++j4)
                dst[j4] = make_float4(R[4 * j4], R[4 * j4 + 1], R[4 * j4 + 2], R[4 * j4 + 3]);
        }
    }

    // the gradient stores (issued by thread 0 and by the first gate thread) have landed
    if (threadIdx.x == 0 || threadIdx.x == 32 * kGateWarp0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, K::TMEM_COLS);
    }
    if (threadIdx.x == 0 && sm.fail) atomicOr(p.err, kErrTimeout);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

constexpr int kMinSegChunks = 4;  // shortest segment worth a CTA of its own

// Segments per head: as many as fill the SMs with one CTA each, none shorter
// than kMinSegChunks chunks.
int bwd_segments(const BwdParams& p) {
    const long long BH = (long long)p.B * p.H;
    const int NC = (p.T + C - 1) / C;
    const int nsm = sm_count();
    long long P = BH < nsm ? nsm / BH : 1;
    if (P > NC / kMinSegChunks) P = NC / kMinSegChunks;
    return P < 1 ? 1 : (int)P;
}

struct WsLayout {
    int P;
    size_t states, oscr, flags, simt, seg_st, seg_ld, seg_flag, total;
};

WsLayout ws_layout(const BwdParams& p) {
    WsLayout w;
    const size_t bh = (size_t)p.B * p.H, nc = (size_t)(p.T + C - 1) / C;
    w.P = bwd_segments(p);
    w.states = p.saved ? 0 : align256(bh * nc * p.dk * p.dv * 4);
    w.oscr = p.saved ? 0 : align256(bh * (size_t)p.T * p.dv * 2);
    w.flags = align256(bh * 4);
    w.simt = align256(simt_bwd_workspace(p));
    // segment exchange, indexed by segment (slot 0 unused)
    w.seg_st = w.P > 1 ? align256((size_t)w.P * bh * p.dk * p.dv * 4) : 0;
    w.seg_ld = w.P > 1 ? align256((size_t)w.P * bh * p.dk * 4) : 0;
    w.seg_flag = w.P > 1 ? align256((size_t)w.P * bh * 4) : 0;
    w.total = w.states + w.oscr + w.flags + w.simt + w.seg_st + w.seg_ld + w.seg_flag;
    return w;
}

template <int DV, bool PRE>
cudaError_t launch_dv(const BwdParams& p, const float* saved, int* flags, const WsLayout& w,
                      cudaStream_t s) {
    BwdKernelArgs a;
    a.p = p;
    a.p.saved = saved;
    a.flags = flags;
    const uint64_t BH = (uint64_t)p.B * p.H;
    if (!make_tmap_bf16_3d(&a.mq, p.q, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mk, p.k, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mg, p.g, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mt, p.tau, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mv, p.v, DV, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mb, p.beta, DV, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdo, p.dO, DV, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdq, p.dq, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdk, p.dk_, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdg, p.dg, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdt, p.dtau, DK, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdv, p.dv_, DV, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mdb, p.dbeta, DV, p.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(BwdSmem<DV>) + 1024;
    auto kern = tc_bwd_kernel<DV, PRE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    char* seg = static_cast<char*>(p.ws) + w.states + w.oscr + w.flags + w.simt;
    for (int P = w.P;; P = 1) {
        a.seg.P = P;
        a.seg.tag = next_launch_tag();
        a.seg.st = P > 1 ? reinterpret_cast<float*>(seg) : nullptr;
        a.seg.ld = P > 1 ? reinterpret_cast<float*>(seg + w.seg_st) : nullptr;
        a.seg.flag = P > 1 ? reinterpret_cast<unsigned*>(seg + w.seg_st + w.seg_ld) : nullptr;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(BH * P));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeCooperative;  // segments wait on one another
        at[0].val.cooperative = 1;
        cfg.attrs = at;
        cfg.numAttrs = P > 1 ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, kern, a);
        if (e != cudaErrorCooperativeLaunchTooLarge || P == 1) return e;
        (void)cudaGetLastError();  // the CTAs do not all fit at once: run unsegmented
    }
}

}  // namespace

bool tc_bwd_supported(const BwdParams& p) {
    return p.bf16 && p.chunk == C && p.T >= 1 && p.dk == DK && (p.dv == 64 || p.dv == 128);
}

size_t tc_bwd_workspace(const BwdParams& p) { return ws_layout(p).total; }

cudaError_t launch_tc_bwd(const BwdParams& p, cudaStream_t s) {
    if (!tc_bwd_supported(p)) return cudaErrorNotSupported;
    const WsLayout w = ws_layout(p);
    char* ws = static_cast<char*>(p.ws);
    const float* saved = p.saved;
    cudaError_t e;
    if (!saved) {
        // recompute the chunk-start states with the forward kernel
        SeqParams f{};  // no workspace: one CTA per sequence
        f.B = p.B; f.H = p.H; f.T = p.T; f.dk = p.dk; f.dv = p.dv; f.chunk = p.chunk; f.bf16 = 1;
        f.q = p.q; f.k = p.k; f.v = p.v; f.g = p.g; f.tau = p.tau; f.beta = p.beta; f.S0 = p.S0;
        f.o = ws + w.states;
        f.ST = nullptr;
        f.saved = reinterpret_cast<float*>(ws);
        f.err = p.err;
        f.preact = p.preact;
        f.wait_limit = p.wait_limit;
        f.withhold_flags = p.withhold_flags;
        if ((e = launch_tc_fwd(f, s)) != cudaSuccess) return e;
        saved = f.saved;
    }
    int* flags = reinterpret_cast<int*>(ws + w.states + w.oscr);
    if ((e = cudaMemsetAsync(flags, 0, (size_t)p.B * p.H * 4, s)) != cudaSuccess) return e;
    if (p.preact)
        e = p.dv == 64 ? launch_dv<64, true>(p, saved, flags, w, s) : launch_dv<128, true>(p, saved, flags, w, s);
    else
        e = p.dv == 64 ? launch_dv<64, false>(p, saved, flags, w, s) : launch_dv<128, false>(p, saved, flags, w, s);
    if (e != cudaSuccess) return e;
    // heads whose decay span needs narrower windows: exact CUDA-core backward
    BwdParams q = p;
    q.ws = ws + w.states + w.oscr + w.flags;
    q.ws_bytes = w.simt;
    return launch_simt_bwd_flagged(q, flags, s);
}

}  // namespace rdm
