// tc_fwd.cu -- chunkwise-parallel DDTS forward on the sm_100a tensor cores.
//
// Rodimus trains the DDTS recurrence chunk by chunk (paperhub.cn rebuttal,
// answer to Q2 and "Efficient Parallelization": selection only along d_k makes
// the chunkwise form possible).  Per (b,h) and chunk of C = 64 tokens, with
// b_t the inclusive running sum of log(alpha) = -g*tau inside the window and
// m a per-channel reference (half the window's total, m = b_last / 2):
//
//   Qt = q * exp(b_t - m)              Kt = k * alpha_hat * exp(m - b_s)
//   A  = mask_{s<=t}(Qt Kt^T)          Vh = beta_hat * v
//   o  = A Vh + Qt (diag(exp(m)) S_prev)                 (intra + inter chunk)
//   S  = diag(exp(b_last)) S_prev + diag(exp(b_last - m)) Kt^T Vh
//
// b_t runs over [b_last, 0] (every log decay is <= 0), so every factor stays
// inside exp(+-|b_last|/2), and products are exact in fp32 range whenever
// |b_last| <= kSpanMax.  A chunk with a larger total is processed as windows of
// 16 tokens, or of 1 token, each window being one pass of the same pipeline
// (exact for any decay).  (The midpoint of the b range is a slightly tighter
// reference but needs b at the window's first token, one more shuffle per
// channel: measured 10% slower on the d_k = 128 long-context forward.)
//
// Sequence segments.  When the (b,h) x d_v-slice units do not fill the GPU,
// each unit's chunks are cut into P contiguous segments, one CTA each.  The
// state map of a segment is affine, S_out = diag(D) S_in + S_loc, with D the
// product of its decays and S_loc its state from a zero start.  A segment
// first computes S_loc alone (no Qt, A or o): with G_s the running sum of
// log(alpha) over the segment, S_loc = sum_s (k_s alpha_hat_s exp(G_end - G_s))
// (beta_hat_s v_s)^T, every factor <= 1, so the products of all its chunks
// accumulate into one tensor-memory sum (chunks taken last to first, which
// gives G_end - G_s as a running sum).  The chunks before the last segment are
// the ones whose maps are needed; that state-only work is shared equally by all
// P CTAs (range j by segment j's CTA, cut in two where a segment boundary falls
// inside it), so every CTA starts its full pass after (P-1)/P of a segment.
// Each piece's (S_loc, log2 D) goes through global memory; a CTA folds the
// pieces before its segment onto S_0 to obtain its true entry state and runs
// the full forward over its chunks.  All CTAs of such a launch are resident
// together (cooperative launch), and every cross-CTA wait is bounded.
//
// One CTA owns one (b,h), a d_v slice of DVT columns and a segment.  Roles:
//   warps 0-7   epilogue: A -> masked bf16 operand, state (fp32 registers),
//               S_hat operand, o store (TMEM lanes = rows; the two warps of a
//               sub-partition take different columns)
//   warps 8-15  gates: TMA tiles -> log-decay scan, Qt, Kt, Vh operands (bf16)
//   warp  16    TMA producer (q, k, g, tau, v, beta tiles, 128B-swizzled)
//   warp  17    TMEM allocator and single-thread tcgen05.mma issuer
// All hand-offs are mbarriers with bounded waits (a timeout sets the device
// status word and the CTA exits cleanly).
#include <cuda.h>

#include <type_traits>

#include "launch.h"
#include "rdm_common.cuh"
#include "tc_common.cuh"

namespace rdm {
namespace {
using namespace tc;

constexpr int C = 64;          // tokens per chunk (tile rows)
constexpr int kEpiWarps = 8;   // two per SM sub-partition
constexpr int kGateWarps = 8;  // two per SM sub-partition
constexpr int kThreads = 32 * (kEpiWarps + kGateWarps + 2);
constexpr int kEpiWarp0 = 0, kGateWarp0 = kEpiWarps, kProdWarp = kEpiWarps + kGateWarps,
              kMmaWarp = kProdWarp + 1;
constexpr int kBarGate = 3;        // named barrier of the gate warps
constexpr int kBarEpi = 4;         // named barrier of the epilogue warps
constexpr int kMinSegChunks = 4;   // shortest segment worth a CTA of its own
constexpr int kMaxSeg = 160;       // most segments per sequence
constexpr int kAhead = 2;          // L2 prefetch distance of the producer, in passes
// low-rank beta_hat: the factor u is read as 16 columns (ranks below 16 come
// zero-filled from TMA, with zero rows of w_up): a 64 x 16 bf16 tile
constexpr int kLrMax = 16;
constexpr int kLrTileBytes = 64 * kLrMax * 2;

template <int DK, int DVT>
struct Cfg {
    static constexpr int NS = DK == 128 ? 1 : 2;   // raw TMA stages
    static constexpr int NB = 2;                   // operand buffers
    static constexpr int KB = DK / 64;             // boxes per key-side tile
    static constexpr int VB = DVT / 64;            // boxes per value-side tile
    static constexpr int RAWK = 4 * KB * kBox;  // q, k, g, tau (NS stages)
    static constexpr int RAWV = 2 * VB * kBox;  // v, beta (one stage, released early)
    static constexpr int G = DK / 8;               // 8-channel groups
    // A | dS | O (double-buffered: the epilogue reads O of one chunk while the
    // tensor core writes the next)
    static constexpr int COL_A = 0, COL_S = 64, COL_O = 64 + DVT;
    static constexpr int TMEM_COLS = (64 + 3 * DVT) <= 256 ? 256 : 512;
    static constexpr bool STAGE_SAVED = DK == 64 && DVT == 64;
};

// info[] of an operand slot
enum { kInfoChunk, kInfoW0, kInfoW1, kInfoLast, kInfoPhase, kInfoP1Last, kInfoPass, kInfoN };

template <int DK, int DVT>
struct alignas(1024) FwdSmem {
    using K = Cfg<DK, DVT>;
    uint8_t raw[K::NS][K::RAWK];
    uint8_t rawv[K::RAWV];
    uint8_t ostage[C * DVT * 2];  // o tile for the TMA store, 128B-swizzled boxes
    // chunk-start state [DK][DVT] fp32 for the TMA store of the saved states
    // (32-column 128B-swizzled boxes; where shared memory allows)
    uint8_t sstage[K::STAGE_SAVED ? DK * DVT * 4 : 16];
    uint8_t qt[K::NB][K::G * kQK];
    uint8_t kt[K::NB][K::G * kQK];
    uint8_t vh[K::NB][C * DVT * 2];
    uint8_t abf[C * C * 2];
    uint8_t shat[DK * DVT * 2];
    float em[K::NB][DK], cf[K::NB][DK], gm[K::NB][DK];
    int info[K::NB][kInfoN];
    uint64_t raw_full[K::NS], raw_empty[K::NS], v_full, v_empty, ops_full[K::NB], ops_empty[K::NB];
    uint64_t mma1_done, as_free, abf_full, mmao_done[2], o_free[2], vh_full[K::NB];
    int need16[2], need1[2];
    int epi_fail;  // the epilogue's own exit decision (written before a role barrier)
    int nbefore;                   // state-only pieces before this CTA's segment
    uint16_t blist[2 * kMaxSeg];   // their slots, in chunk order
    uint8_t before[2 * kMaxSeg];  // state-only pieces that precede this CTA's segment
    uint32_t tmem_base;
    int fail;
};

// Segment s covers chunks [seg_start(s), seg_start(s+1)).
__host__ __device__ inline int seg_start(int s, int NC, int P) {
    const unsigned long long x = (unsigned long long)s * (unsigned)NC;
    return x <= 0xffffffffull ? (int)((unsigned)x / (unsigned)P) : (int)(x / (unsigned)P);
}
// State-only range [a0, a1) of segment j's CTA: the P-th part j of the chunks
// before the last segment.  `mid` is the segment boundary strictly inside it
// (a1 when none); the pieces are [a0, mid) (slot 2j) and [mid, a1) (slot 2j+1).
struct P1Range {
    int a0, a1, mid;
};
// (kept out of line: the integer divisions stay out of the role loops' code)
__host__ __device__ __noinline__ P1Range p1_range(int j, int NC, int P) {
    const int n1 = seg_start(P - 1, NC, P);
    P1Range r;
    r.a0 = seg_start(j, n1, P);
    r.a1 = seg_start(j + 1, n1, P);
    r.mid = r.a1;
    for (int s = P - 1; s >= 1; --s) {
        const int cs = seg_start(s, NC, P);
        if (cs > r.a0 && cs < r.a1) r.mid = cs;
    }
    return r;
}
// true when no state-only range holds two segment boundaries (each range is
// then at most two pieces)
bool p1_ranges_ok(int NC, int P) {
    for (int j = 0; j < P; ++j) {
        const P1Range r = p1_range(j, NC, P);
        int inside = 0;
        for (int s = 1; s < P; ++s) {
            const int cs = seg_start(s, NC, P);
            inside += cs > r.a0 && cs < r.a1;
        }
        if (inside > 1 || r.a1 <= r.a0) return false;
    }
    return true;
}

// Segment exchange area (global): per (piece slot < 2P, unit) the local state
// [DK][DVT] and log2 of the decay product per channel, and a flag that holds
// `epoch` once those are written.
struct SegArgs {
    int P;
    unsigned epoch;
    float* st;
    float* ld;
    unsigned* flag;
};

struct FwdKernelArgs {
    CUtensorMap mq, mk, mg, mt, mv, mb, mo;
    CUtensorMap mu;  // low-rank beta_hat factor u [B][T][r] as boxes of 16 columns x 64 tokens
    CUtensorMap msv;  // saved states as [rows = B*H*NC*DK][dv] fp32 (when staged)
    SeqParams p;
    SegArgs seg;
};

// PRE: g, tau, beta arrive before their activations; FEED: o_t += d (.) v_t;
// LR: beta_hat's pre-activation is u_t . w_up[h] (rank r <= 16), built on chip
template <int DK, int DVT, bool PRE, bool FEED, bool LR>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdKernelArgs A) {
    using K = Cfg<DK, DVT>;
    constexpr int NS = K::NS, NB = K::NB, KB = K::KB, VB = K::VB;
    // Who builds Vh = beta_hat * v: the epilogue warps when d_k = 128 (the gate
    // warps then carry twice the key-side work and are the slower role, which
    // also hides the v / beta load behind them) and when the gates arrive before
    // their activations (the gate warps then also evaluate softplus and sigmoid
    // on the key side; measured 124 -> 116 us on the 130M-scale layer); the gate
    // warps otherwise, where moving it would put that load on the epilogue's
    // path to the first MMA group.
    constexpr bool kVhEpi = DK == 128 || PRE;
    // align by pointer arithmetic on the __shared__ array so that every access
    // below stays a shared-memory access (an integer round trip would make it generic)
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    FwdSmem<DK, DVT>& sm = *reinterpret_cast<FwdSmem<DK, DVT>*>(
        smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
    const SeqParams& p = A.p;
    const SegArgs& sg = A.seg;
    const long long WL = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;  // bound of every wait
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NJ = p.dv / DVT;
    const int units = p.B * p.H * NJ;
    const int unit = blockIdx.x % units, seg = blockIdx.x / units;
    const int bh = unit / NJ, j0 = (unit % NJ) * DVT;
    const int T = p.T, NC = (T + C - 1) / C;
    const int NCS = (T + p.chunk - 1) / p.chunk;  // saved chunk-start states per sequence
    const int P = sg.P;
    const int c0 = seg_start(seg, NC, P), c1 = seg_start(seg + 1, NC, P);
    const int nseg = c1 - c0;
    // state-only range of this CTA (none when P == 1)
    const P1Range g1 = P > 1 ? p1_range(seg, NC, P) : P1Range{0, 0, 0};
    const int nP1 = g1.a1 - g1.a0;
    const bool has_p1 = nP1 > 0, split1 = g1.mid < g1.a1;
    const int nL = nP1 + nseg;  // chunk passes
    // pass li: phase 1 (state only, chunks a1-1 down to a0) for the first nP1
    // passes, then phase 2 (the segment's chunks in order)
    auto pass_chunk = [&](int li) { return li < nP1 ? g1.a1 - 1 - li : c0 + li - nP1; };
    auto pass_p2 = [&](int li) { return li >= nP1; };
    // state-only chunks that open / close a piece (in processing order)
    auto piece_open = [&](int c) { return c == g1.a1 - 1 || (split1 && c == g1.mid - 1); };
    auto piece_close = [&](int c) { return c == g1.a0 || (split1 && c == g1.mid); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.raw_full[s], 1);
            mbar_init(&sm.raw_empty[s], kGateWarps);
        }
        mbar_init(&sm.v_full, 1);
        mbar_init(&sm.v_empty, kGateWarps);
        for (int b = 0; b < NB; ++b) {
            mbar_init(&sm.ops_full[b], kGateWarps);
            mbar_init(&sm.ops_empty[b], 1 + kEpiWarps);
        }
        mbar_init(&sm.mma1_done, 1);
        mbar_init(&sm.as_free, kEpiWarps);
        mbar_init(&sm.abf_full, kEpiWarps);
        mbar_init(&sm.mmao_done[0], 1);
        mbar_init(&sm.mmao_done[1], 1);
        mbar_init(&sm.o_free[0], kEpiWarps);
        mbar_init(&sm.o_free[1], kEpiWarps);
        for (int b = 0; b < NB; ++b) mbar_init(&sm.vh_full[b], kEpiWarps);
        sm.epi_fail = 0;
        sm.need16[0] = sm.need16[1] = sm.need1[0] = sm.need1[1] = 0;
        sm.fail = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, K::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_tmap(&A.mq); prefetch_tmap(&A.mk); prefetch_tmap(&A.mg);
        prefetch_tmap(&A.mt); prefetch_tmap(&A.mv); prefetch_tmap(&A.mo);
        prefetch_tmap(LR ? &A.mu : &A.mb);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* fail = &sm.fail;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0, issued_v = 0;
            for (int li = 0; li < nL; ++li) {
                const int st = li % NS, c = pass_chunk(li);
                const bool p2 = pass_p2(li);
                if (li >= NS && !mbar_wait(&sm.raw_empty[st], ((li / NS) - 1) & 1, fail, WL))
                    break;
                // the state-only pass does not read q
                mbar_expect_tx(&sm.raw_full[st], K::RAWK - (p2 ? 0 : KB * kBox));
                uint8_t* raw = sm.raw[st];
                for (int kb = 0; kb < KB; ++kb) {
                    if (p2)
                        tma_load_3d(raw + (0 * KB + kb) * kBox, &A.mq, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (1 * KB + kb) * kBox, &A.mk, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (2 * KB + kb) * kBox, &A.mg, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (3 * KB + kb) * kBox, &A.mt, &sm.raw_full[st], 64 * kb, c * C, bh);
                }
                ++issued;
                // the tiles of the pass kAhead further on, into L2
                if (li + kAhead < nL) {
                    const int ca = pass_chunk(li + kAhead);
                    const bool qa = pass_p2(li + kAhead);
                    for (int kb = 0; kb < KB; ++kb) {
                        if (qa) tma_prefetch_3d(&A.mq, 64 * kb, ca * C, bh);
                        tma_prefetch_3d(&A.mk, 64 * kb, ca * C, bh);
                        tma_prefetch_3d(&A.mg, 64 * kb, ca * C, bh);
                        tma_prefetch_3d(&A.mt, 64 * kb, ca * C, bh);
                    }
                    for (int vb = 0; vb < VB; ++vb) {
                        tma_prefetch_3d(&A.mv, j0 + 64 * vb, ca * C, bh);
                        if constexpr (!LR) tma_prefetch_3d(&A.mb, j0 + 64 * vb, ca * C, bh);
                    }
                }
                if (li >= 1 && !mbar_wait(&sm.v_empty, (li - 1) & 1, fail, WL)) break;
                mbar_expect_tx(&sm.v_full, LR ? VB * kBox + kLrTileBytes : K::RAWV);
                for (int vb = 0; vb < VB; ++vb) {
                    tma_load_3d(sm.rawv + vb * kBox, &A.mv, &sm.v_full, j0 + 64 * vb, c * C, bh);
                    if constexpr (!LR)
                        tma_load_3d(sm.rawv + (VB + vb) * kBox, &A.mb, &sm.v_full, j0 + 64 * vb, c * C, bh);
                }
                // the u rows of the chunk's tokens into the (otherwise unused) beta space
                if constexpr (LR) tma_load_3d(sm.rawv + VB * kBox, &A.mu, &sm.v_full, 0, c * C, bh / p.H);
                ++issued_v;
            }
            // never leave the CTA with copies in flight
            for (int li = issued - NS < 0 ? 0 : issued - NS; li < issued; ++li)
                drain_wait(&sm.raw_full[li % NS], (li / NS) & 1);
            if (issued_v > 0) drain_wait(&sm.v_full, (issued_v - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tA = tmem + K::COL_A, tS = tmem + K::COL_S, tO = tmem + K::COL_O;
            constexpr uint32_t id1 = idesc_bf16(64, 64, 0, 0);    // A  = Qt Kt^T
            constexpr uint32_t idS = idesc_bf16(DK, DVT, 1, 1);   // dS = Kt^T Vh
            constexpr uint32_t idO = idesc_bf16(64, DVT, 0, 1);   // O  = A Vh + Qt S_hat
            // io counts the items that produce o, nas the waits for the epilogue to
            // release A and dS (before every item that starts dS from zero, but the
            // first item of the launch; a state-only piece accumulates into dS)
            int item = 0, n1 = 0, io = 0, nas = 0;
            while (true) {
                const int ob = item % NB;
                if (!mbar_wait(&sm.ops_full[ob], (item / NB) & 1, fail, WL)) break;
                const int last = sm.info[ob][kInfoLast];
                const bool p2 = sm.info[ob][kInfoPhase] == 2;
                const bool p1last = sm.info[ob][kInfoP1Last];
                const bool fresh = p2 || piece_open(sm.info[ob][kInfoChunk]);
                if constexpr (kVhEpi)
                    if (!mbar_wait(&sm.vh_full[ob], (item / NB) & 1, fail, WL)) break;
                if (fresh && item > 0) {
                    if (!mbar_wait(&sm.as_free, nas & 1, fail, WL)) break;
                    ++nas;
                }
                tc_fence_after();
                const uint32_t q = smem_u32(sm.qt[ob]) >> 4, k = smem_u32(sm.kt[ob]) >> 4;
                const uint32_t v = smem_u32(sm.vh[ob]) >> 4;
                if (p2) {
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks)
                        mma_bf16_w(tA, q + sd_lo(ks * 2 * kQK, kQK), sd_hi(128),
                                   k + sd_lo(ks * 2 * kQK, kQK), sd_hi(128), id1, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16_w(tS, k + sd_lo(ks * 256, 128), sd_hi(kQK), v + sd_lo(ks * 256, 128),
                               sd_hi(1024), idS, ks > 0 || !fresh);
                if (p2 || p1last) {
                    mma_commit(&sm.mma1_done);
                    ++n1;
                }
                if (p2) {
                    if (!mbar_wait(&sm.abf_full, io & 1, fail, WL)) break;
                    const int obuf = io & 1;
                    if (io >= 2 && !mbar_wait(&sm.o_free[obuf], ((io >> 1) - 1) & 1, fail, WL))
                        break;
                    tc_fence_after();
                    const uint32_t a = smem_u32(sm.abf) >> 4, sh = smem_u32(sm.shat) >> 4;
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        mma_bf16_w(tO + obuf * DVT, a + sd_lo(ks * 2048, 1024), sd_hi(128),
                                   v + sd_lo(ks * 256, 128), sd_hi(1024), idO, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks)
                        mma_bf16_w(tO + obuf * DVT, q + sd_lo(ks * 2 * kQK, kQK), sd_hi(128),
                                   sh + sd_lo(ks * 256, 128), sd_hi(DK * 16), idO, 1);
                    mma_commit(&sm.mmao_done[obuf]);
                    ++io;
                }
                mma_commit(&sm.ops_empty[ob]);
                if (last) break;
                ++item;
            }
            // let issued MMAs finish before TMEM is released
            if (n1 > 0) drain_wait(&sm.mma1_done, (n1 - 1) & 1);
            if (io > 0) drain_wait(&sm.mmao_done[(io - 1) & 1], ((io - 1) >> 1) & 1);
        }
        __syncwarp();
    } else if (warp >= kGateWarp0) {
        // ------------------------------------------------------------ gates
        // warp gw owns channel groups [gw*GW, gw*GW + GW) (8 channels each) for all
        // 64 tokens; lane -> (group cgl, segment of SEGT consecutive tokens).  The
        // running sum of log(alpha) is an in-thread scan plus a shuffle scan over
        // the segments: no data crosses warps.  The chunk is cut into windows of W
        // tokens (64, or 16 / 1 when the decay span is too wide for one
        // reference); only that choice is agreed across the gate warps.
        constexpr int G = K::G, GW = G / kGateWarps, NSW = 32 / GW, SEGT = C / NSW;
        constexpr int VG = DVT / 8, TPG = 32 * kGateWarps / VG, VIT = C / TPG;
        const int gw = warp - kGateWarp0, gt = gw * 32 + lane;
        const int cgl = lane % GW, seg_l = lane / GW;
        const int cg = gw * GW + cgl;
        const int tb = seg_l * SEGT;  // first token of my segment
        const uint32_t full = 0xffffffffu;
        const int W0 = p.chunk;  // window width asked for: 64, 32 or 16 tokens
        int item = 0;
        float gt2[8];  // state-only pass: log2 decay of the chunks after the current one
#pragma unroll
        for (int e = 0; e < 8; ++e) gt2[e] = 0.0f;
        // one pass over a chunk; kP2 selects the full pass at compile time (so the
        // state-only pass's registers are free in the other); false stops the role
        auto pass = [&](int li, auto kP2) -> bool {
            const int st = li % NS, c = pass_chunk(li);
            constexpr bool p2 = decltype(kP2)::value;
            if (!mbar_wait_own(&sm.raw_full[st], (li / NS) & 1, fail, WL)) return false;
            const uint8_t* raw = sm.raw[st];
            const int nval = min(C, T - c * C);
            // log2(alpha_hat) of my tokens is kept from the scan for the operand pass
            // when registers allow (d_k = 64); otherwise that pass re-reads g and tau
            constexpr bool kKeepLah = SEGT <= 2;
            float b[SEGT][8], bl[8];
            [[maybe_unused]] float lah2[kKeepLah ? SEGT : 1][8];
            // window-relative inclusive running sum of log(alpha) over my tokens, and
            // b at the last valid token of my window (W in {64, 32, 16})
            auto scan = [&](int W) {
#pragma unroll
                for (int u = 0; u < SEGT; ++u) {
                    float g8[8], t8[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(tb + u, cg)), g8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(tb + u, cg)), t8);
                    if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float la = (tb + u < nval) ? log_alpha(g8[e], t8[e]) : 0.0f;
                        b[u][e] = (u == 0 || W == 1) ? la : b[u - 1][e] + la;
                        if constexpr (kKeepLah)
                            lah2[u][e] = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                    }
                }
                if (W == 1) return;
                const int WLN = W / SEGT * GW;       // lanes per window
                const int l0 = lane & ~(WLN - 1);    // first lane of my window
                const int tw0 = (l0 / GW) * SEGT;    // first token of my window
                const int tl = min(tw0 + W, nval) - 1;  // last valid token of my window
                const int lsrc = cgl + GW * (max(tl, tw0) / SEGT);
                const int usrc = max(tl, tw0) % SEGT;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float tot = b[SEGT - 1][e];
                    float x = tot;
#pragma unroll
                    for (int d = GW; d < 32; d <<= 1) {
                        const float y = __shfl_up_sync(full, x, d);
                        if ((lane & (WLN - 1)) >= d) x += y;
                    }
                    const float excl = x - tot;
                    float mine = 0.0f;
#pragma unroll
                    for (int u = 0; u < SEGT; ++u) {
                        b[u][e] += excl;
                        if (u == usrc) mine = b[u][e];
                    }
                    bl[e] = __shfl_sync(full, mine, lsrc);
                }
            };
            // true when some window of this chunk spans more log-decay than one
            // reference holds; every gate warp takes the same answer
            auto too_wide = [&](int* flag) {
                float span = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) span = fmaxf(span, -bl[e]);
                if (tb >= nval) span = 0.0f;
                if (__any_sync(full, !(span <= kSpanMax)) && lane == 0) *flag = li + 1;
                named_bar(kBarGate, 32 * kGateWarps);
                return *flag == li + 1;
            };
            // Vh = beta_hat * v for the rows of [w0, w1), zero elsewhere
            bool have_v = false;
            auto write_vh = [&](int ob, int w0, int w1) {
                if constexpr (kVhEpi) return;
                if (!have_v) {
                    have_v = mbar_wait_own(&sm.v_full, li & 1, fail, WL);
                    if (!have_v) return;
                }
#pragma unroll
                for (int it = 0; it < VIT; ++it) {
                    const int jg = gt / TPG, t = (gt % TPG) + TPG * it;
                    const bool in = t >= w0 && t < w1;
                    const uint4 v8 = *reinterpret_cast<const uint4*>(sm.rawv + off_raw(t, jg));
                    const uint4 b8 = *reinterpret_cast<const uint4*>(sm.rawv + VB * kBox + off_raw(t, jg));
                    uint4 o8 = make_uint4(0u, 0u, 0u, 0u);
                    if constexpr (PRE) {
                        float vf[8], bf8[8], of[8];
                        unpack8(v8, vf);
                        unpack8(b8, bf8);
                        activate_beta8(bf8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) of[e] = vf[e] * bf8[e];
                        if (in) o8 = pack8(of);
                    } else {
                        if (in) o8 = bmul8(v8, b8);
                    }
                    *reinterpret_cast<uint4*>(sm.vh[ob] + off_vh(t, jg * 8)) = o8;
                }
            };
            auto publish = [&](int ob, int w0, int w1) {
                if (gt == 0) {
                    const bool end = p2 ? (c == c1 - 1) && (w1 == nval) : piece_close(c);
                    sm.info[ob][kInfoChunk] = c;
                    sm.info[ob][kInfoW0] = w0;
                    sm.info[ob][kInfoW1] = w1;
                    sm.info[ob][kInfoLast] = p2 && end;
                    sm.info[ob][kInfoPhase] = p2 ? 2 : 1;
                    sm.info[ob][kInfoP1Last] = !p2 && end;
                    if constexpr (kVhEpi) sm.info[ob][kInfoPass] = li;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.ops_full[ob]);
            };
            if constexpr (!p2) {
                // ---- state-only pass (chunks last to first, all of them whole):
                // Kt = k alpha_hat exp(G_end - G_s) with G_end the end of the piece,
                // G_end - G_s = gt2 (the decay of the piece's later chunks, log2) +
                // b_last - b_s; every factor <= 1
                if (piece_open(c)) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) gt2[e] = 0.0f;
                }
                scan(C);
                const int ob = item % NB;
                if (item >= NB && !mbar_wait_own(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, WL))
                    return false;
#pragma unroll
                for (int u = 0; u < SEGT; ++u) {
                    const int t = tb + u;
                    float k8[8], lah[8], ok[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 1 * KB * kBox + off_raw(t, cg)), k8);
                    if constexpr (kKeepLah) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) lah[e] = lah2[u][e];
                    } else {
                        float g8[8], t8[8];
                        unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(t, cg)), g8);
                        unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(t, cg)), t8);
                        if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) lah[e] = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        ok[e] = k8[e] * ex2_fast(lah[e] + fmaf(bl[e] - b[u][e], kLog2e, gt2[e]));
                    *reinterpret_cast<uint4*>(sm.kt[ob] + off_qk(t, cg * 8)) = pack8(ok);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) gt2[e] = fmaf(bl[e], kLog2e, gt2[e]);
                // log2 of the piece's decay product, for the epilogue
                if (tb == 0 && piece_close(c)) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) sm.gm[ob][cg * 8 + e] = gt2[e];
                }
                write_vh(ob, 0, C);
                if (!kVhEpi && !have_v) return false;
                publish(ob, 0, C);
                ++item;
            } else {
                // window width: the chunk size asked for (64, 32 or 16 tokens),
                // narrowed to 16 and then to single tokens while some window
                // spans more log-decay than one reference holds
                int W = W0;
                scan(W);
                bool wide = too_wide(&sm.need16[li & 1]);
                if (wide && W > 16) {
                    W = 16;
                    scan(16);
                    wide = too_wide(&sm.need1[li & 1]);
                }
                if (wide) {
                    W = 1;
                    scan(1);
                }
                if (W == C) {
                    // ---- one window = the whole chunk (rows past T hold zeros from the
                    // TMA fill, so every row can be computed unmasked)
                    const int ob = item % NB;
                    if (item >= NB && !mbar_wait_own(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, WL))
                        return false;
                    float mL[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) mL[e] = 0.5f * bl[e] * kLog2e;
#pragma unroll
                    for (int u = 0; u < SEGT; ++u) {
                        const int t = tb + u;
                        float k8[8], lah[8], ok[8];
                        unpack8(*reinterpret_cast<const uint4*>(raw + 1 * KB * kBox + off_raw(t, cg)), k8);
                        if constexpr (kKeepLah) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) lah[e] = lah2[u][e];
                        } else {
                            float g8[8], t8[8];
                            unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(t, cg)), g8);
                            unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(t, cg)), t8);
                            if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                            for (int e = 0; e < 8; ++e) lah[e] = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                        }
                        float q8[8], oq[8];
                        unpack8(*reinterpret_cast<const uint4*>(raw + 0 * KB * kBox + off_raw(t, cg)), q8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float d = fmaf(b[u][e], kLog2e, -mL[e]);
                            oq[e] = q8[e] * ex2_fast(d);
                            ok[e] = k8[e] * ex2_fast(lah[e] - d);
                        }
                        *reinterpret_cast<uint4*>(sm.qt[ob] + off_qk(t, cg * 8)) = pack8(oq);
                        *reinterpret_cast<uint4*>(sm.kt[ob] + off_qk(t, cg * 8)) = pack8(ok);
                    }
                    if (tb == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            sm.em[ob][cg * 8 + e] = ex2_fast(mL[e]);
                            sm.cf[ob][cg * 8 + e] = ex2_fast(bl[e] * kLog2e - mL[e]);
                            sm.gm[ob][cg * 8 + e] = ex2_fast(bl[e] * kLog2e);
                        }
                    }
                    write_vh(ob, 0, C);
                    if (!kVhEpi && !have_v) return false;
                    publish(ob, 0, nval);
                    ++item;
                } else {
                    bool ok_loop = true;
                    for (int w0 = 0; w0 < nval; w0 += W) {
                        const int w1 = min(w0 + W, nval);
                        const int ob = item % NB;
                        if (item >= NB &&
                            !mbar_wait_own(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, WL)) {
                            ok_loop = false;
                            break;
                        }
#pragma unroll 1
                        for (int u = 0; u < SEGT; ++u) {
                            const int t = tb + u;
                            const bool in = t >= w0 && t < w1;
                            float q8[8], k8[8], g8[8], t8[8], oq[8], ok[8];
                            unpack8(*reinterpret_cast<const uint4*>(raw + 0 * KB * kBox + off_raw(t, cg)), q8);
                            unpack8(*reinterpret_cast<const uint4*>(raw + 1 * KB * kBox + off_raw(t, cg)), k8);
                            unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(t, cg)), g8);
                            unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(t, cg)), t8);
                            if constexpr (PRE) activate_gates8(g8, t8);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                // reference m = half the window's total log decay, blast = b at its end
                                const float blast = W == 1 ? b[u][e] : bl[e];
                                const float m = W == 1 ? b[u][e] : 0.5f * bl[e];
                                const float d = (b[u][e] - m) * kLog2e;
                                const float lah = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                                oq[e] = in ? q8[e] * ex2_fast(d) : 0.0f;
                                ok[e] = in ? k8[e] * ex2_fast(lah - d) : 0.0f;
                                if (t == w0) {
                                    sm.em[ob][cg * 8 + e] = ex2_fast(m * kLog2e);
                                    sm.cf[ob][cg * 8 + e] = ex2_fast((blast - m) * kLog2e);
                                    sm.gm[ob][cg * 8 + e] = ex2_fast(blast * kLog2e);
                                }
                            }
                            *reinterpret_cast<uint4*>(sm.qt[ob] + off_qk(t, cg * 8)) = pack8(oq);
                            *reinterpret_cast<uint4*>(sm.kt[ob] + off_qk(t, cg * 8)) = pack8(ok);
                        }
                        write_vh(ob, w0, w1);
                        if (!kVhEpi && !have_v) {
                            ok_loop = false;
                            break;
                        }
                        publish(ob, w0, w1);
                        ++item;
                    }
                    if (!ok_loop) return false;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.raw_empty[st]);
                if constexpr (!kVhEpi) mbar_arrive(&sm.v_empty);
            }
            return true;
        };
        int li = 0;
        bool run = true;
        for (; run && li < nP1; ++li) run = pass(li, std::false_type{});
        for (; run && li < nL; ++li) run = pass(li, std::true_type{});
    } else {
        // ------------------------------------------------------------ epilogue
        // A and O are M = 64 accumulators (TMEM lanes 0-15 of each sub-partition):
        // the split load gives row tA to two threads, lane >> 4 (hf) picking the
        // half of the columns, and the two warps of a sub-partition (eh) take
        // different quarters.  The state is M = DK: split the same way for
        // DK = 64; one row per thread (all 32 lanes), half the columns per warp,
        // for DK = 128.
        constexpr bool kSplitS = DK == 64;
        constexpr int SC = kSplitS ? DVT / 4 : DVT / 2;  // state columns per thread
        constexpr int OC = DVT / 4;                      // o columns per thread
        const int ew = warp - kEpiWarp0, sub = ew & 3, eh = ew >> 2;
        const int hf = lane >> 4;
        const int tA = 16 * sub + (lane & 15);
        const int iS = kSplitS ? tA : 32 * sub + lane;
        const int oc0 = hf * (DVT / 2) + eh * OC;  // first o column of this thread
        const int sc0 = kSplitS ? oc0 : eh * SC;   // first state column of this thread
        const uint32_t lb = (uint32_t)(32 * sub) << 16;
        // SC / OC columns of this thread from a DVT-wide accumulator at `col`
        auto ld_cols = [&](uint32_t col, float* v, bool state) {
            if (state && !kSplitS) {
                if constexpr (SC == 32) tmem_ld32(tmem + lb + col + eh * SC, v);
                else tmem_ld16(tmem + lb + col + eh * SC, v);
            } else {
                if constexpr (OC == 32) tmem_ld32_split<DVT / 2>(tmem + lb + col + eh * OC, v);
                else tmem_ld16_split<DVT / 2>(tmem + lb + col + eh * OC, v);
            }
            tmem_ld_wait();
        };
        float S[SC];
        auto epi_sync = [&]() { named_bar(kBarEpi, 32 * kEpiWarps); };
        auto load_s0 = [&]() {
#pragma unroll
            for (int j = 0; j < SC; ++j)
                S[j] = p.S0 ? p.S0[((size_t)bh * DK + iS) * p.dv + j0 + sc0 + j] : 0.0f;
        };
        // entry state of this segment: S_0 carried through the maps of all the
        // state-only pieces before it, in chunk order, S <- diag(D) S + S_loc
        // A piece's state in the workspace is kept in the epilogue's register
        // order: float4 k of thread et at index k * 256 + et, so that each warp
        // instruction reads or writes 512 contiguous bytes (the rows of the
        // state are 512 bytes apart in the threads' own layout).
        auto piece_ptr = [&](size_t u) {
            return reinterpret_cast<float4*>(sg.st) + u * (DK * DVT / 4) + (threadIdx.x - 32 * kEpiWarp0);
        };
        // which state-only pieces precede this segment (slot 2j + h is [a0, mid)
        // or [mid, a1) of range j), in chunk order: worked out at the start,
        // while the first tiles are still in flight (one slot per thread; the
        // range arithmetic divides 64-bit integers)
        auto plan_fold = [&]() {
            const int et = threadIdx.x - 32 * kEpiWarp0;
            for (int slot = et; slot < 2 * P; slot += 32 * kEpiWarps) {
                const P1Range r = p1_range(slot >> 1, NC, P);
                const int lo = (slot & 1) ? r.mid : r.a0, hi = (slot & 1) ? r.a1 : r.mid;
                sm.before[slot] = lo < hi && hi <= c0;
            }
            epi_sync();
            if (threadIdx.x == 0) {
                int nb = 0;
                for (int slot = 0; slot < 2 * P; ++slot)
                    if (sm.before[slot]) sm.blist[nb++] = (uint16_t)slot;
                sm.nbefore = nb;
            }
            epi_sync();
        };
        // entry state of this segment: S_0 carried through the maps of the pieces
        // before it, S <- diag(D_p) S + S_loc_p in chunk order, evaluated as
        //   S = (prod_p D_p) S_0 + sum_p (prod_{p' after p} D_p') S_loc_p
        // (same products, every piece's loads in flight together)
        auto fold_earlier = [&]() -> bool {
            const int nb = sm.nbefore;
            if (nb == 0) {
                load_s0();
                return true;
            }
            if (threadIdx.x == 0) {
                const long long t0 = clock64();
                for (int i = 0; i < nb && !sm.epi_fail; ++i) {
                    const unsigned* fl = &sg.flag[sm.blist[i] * units + unit];
                    while (ld_acquire_gpu(fl) != sg.epoch)
                        if (clock64() - t0 > WL) {
                            *fail = 1;
                            sm.epi_fail = 1;
                            break;
                        }
                }
            }
            epi_sync();
            if (sm.epi_fail) return false;  // written by thread 0 before the barrier
#pragma unroll
            for (int j = 0; j < SC; ++j) S[j] = 0.0f;
            float lsum = 0.0f;  // log2 of the decay of the pieces after the current one
#pragma unroll 1
            for (int i = nb - 1; i >= 0; --i) {
                const size_t u = (size_t)sm.blist[i] * units + unit;
                const float4* src = piece_ptr(u);
                const float sc = ex2_fast(lsum);
                lsum += __ldcg(&sg.ld[u * DK + iS]);
#pragma unroll
                for (int j4 = 0; j4 < SC / 4; ++j4) {
                    const float4 x = __ldcg(src + j4 * 32 * kEpiWarps);
                    S[4 * j4] = fmaf(sc, x.x, S[4 * j4]);
                    S[4 * j4 + 1] = fmaf(sc, x.y, S[4 * j4 + 1]);
                    S[4 * j4 + 2] = fmaf(sc, x.z, S[4 * j4 + 2]);
                    S[4 * j4 + 3] = fmaf(sc, x.w, S[4 * j4 + 3]);
                }
            }
            if (p.S0) {
                const float d0 = ex2_fast(lsum);
                const float* s0 = p.S0 + ((size_t)bh * DK + iS) * p.dv + j0 + sc0;
#pragma unroll
                for (int j = 0; j < SC; ++j) S[j] = fmaf(d0, s0[j], S[j]);
            }
            return true;
        };
        // publish the map of a state-only piece (S_loc in S, log2 D in ld2)
        auto publish_piece = [&](int slot, float ld2) -> bool {
            const size_t u = (size_t)slot * units + unit;
            float4* dst = piece_ptr(u);
#pragma unroll
            for (int j4 = 0; j4 < SC / 4; ++j4)
                dst[j4 * 32 * kEpiWarps] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
            if (sc0 == 0) sg.ld[u * DK + iS] = ld2;
            // every row is written (CTA barrier); one fence at GPU scope then makes
            // all of them visible before the flag is
            epi_sync();
            if (threadIdx.x == 0 && !p.withhold_flags) {
                __threadfence();
                st_release_gpu(&sg.flag[u], sg.epoch);
            }
            return true;
        };
        // o rows [w0, w1) of chunk c from the O buffer of o-item `io`.  A whole
        // chunk goes out through the staging tile and one TMA store (rows past T
        // are clipped by the TMA unit); a window writes its rows directly.
        auto store_o = [&](int io, int c, int w0, int w1) -> bool {
            const int obuf = io & 1;
            if (!mbar_wait_own(&sm.mmao_done[obuf], (io >> 1) & 1, fail, WL)) return false;
            tc_fence_after();
            float v[OC];
            ld_cols(K::COL_O + obuf * DVT, v, false);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.o_free[obuf]);
            // feedthrough o_t += d (.) v_t (row tA, this thread's columns); v of
            // this chunk has left shared memory, its rows come back from L2
            if (FEED && c * C + tA < T) {
                const uint4* vr = reinterpret_cast<const uint4*>(
                    static_cast<const __nv_bfloat16*>(p.v) + ((size_t)bh * T + (size_t)c * C + tA) * p.dv + j0 + oc0);
                const float4* dr = reinterpret_cast<const float4*>(p.dfeed + (size_t)(bh % p.H) * p.dv + j0 + oc0);
#pragma unroll
                for (int s8 = 0; s8 < OC / 8; ++s8) {
                    float x[8];
                    unpack8(__ldg(vr + s8), x);
                    const float4 d0 = __ldg(dr + 2 * s8), d1 = __ldg(dr + 2 * s8 + 1);
                    const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[8 * s8 + e] = fmaf(dd[e], x[e], v[8 * s8 + e]);
                }
            }
            const bool whole = w0 == 0 && w1 == min(C, T - c * C);
            if (whole) {
                // the previous store has read the staging tile
                if (threadIdx.x == 0) bulk_wait_read_all();
                epi_sync();
#pragma unroll
                for (int s8 = 0; s8 < OC / 8; ++s8)
                    *reinterpret_cast<uint4*>(sm.ostage + off_raw(tA, (oc0 >> 3) + s8)) = pack8(v + 8 * s8);
                fence_proxy_async_smem();
                epi_sync();
                if (threadIdx.x == 0) {
#pragma unroll
                    for (int vb = 0; vb < VB; ++vb)
                        tma_store_3d(&A.mo, sm.ostage + vb * kBox, j0 + 64 * vb, c * C, bh);
                    bulk_commit();
                }
            } else if (tA >= w0 && tA < w1) {
                __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) +
                                      ((size_t)bh * T + (size_t)c * C + tA) * p.dv + j0 + oc0;
#pragma unroll
                for (int s8 = 0; s8 < OC / 8; ++s8)
                    reinterpret_cast<uint4*>(orow)[s8] = pack8(v + 8 * s8);
            }
            return true;
        };
        if constexpr (LR) {
            // w_up[h][:, j0 .. j0 + DVT) as float32 [16][DVT] beside the u tile
            // (rows r .. 15 zero), staged once for all chunks
            float* wsm = reinterpret_cast<float*>(sm.rawv + VB * kBox + kLrTileBytes);
            const int et = threadIdx.x - 32 * kEpiWarp0, hh = bh % p.H;
            for (int i = et; i < kLrMax * DVT; i += 32 * kEpiWarps) {
                const int rho = i / DVT, j = i % DVT;
                wsm[i] = rho < p.beta_rank ? p.beta_w[((size_t)hh * p.beta_rank + rho) * p.dv + j0 + j] : 0.0f;
            }
            epi_sync();
        }
        bool ok_run = true;
        if (P == 1) {
            load_s0();
        } else {
            plan_fold();
            if (!has_p1) ok_run = fold_earlier();
        }
        int item = 0, io = 0, nm1 = 0, pc = 0, pw0 = 0, pw1 = 0;
        while (ok_run) {
            const int ob = item % NB;
            if (!mbar_wait_own(&sm.ops_full[ob], (item / NB) & 1, fail, WL)) break;
            const int c = sm.info[ob][kInfoChunk], w0 = sm.info[ob][kInfoW0], w1 = sm.info[ob][kInfoW1];
            const int last = sm.info[ob][kInfoLast], p1last = sm.info[ob][kInfoP1Last];
            const bool p2 = sm.info[ob][kInfoPhase] == 2;
            if constexpr (kVhEpi) {
                // Vh = beta_hat * v for the rows of [w0, w1), zero elsewhere; the slot is
                // free once the tensor core has finished the item NB back
                const int li = sm.info[ob][kInfoPass];
                const int nval = min(C, T - c * C);
                if (!mbar_wait_own(&sm.v_full, li & 1, fail, WL)) break;
                if (item >= NB && !mbar_wait_own(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, WL))
                    break;
                const int et = threadIdx.x - 32 * kEpiWarp0;
                // LR: this thread's token (the same for every item below) and its
                // row of the u tile
                float ur[LR ? kLrMax : 1];
                if constexpr (LR) {
                    const uint8_t* urow = sm.rawv + VB * kBox + (et % C) * (kLrMax * 2);
                    unpack8(*reinterpret_cast<const uint4*>(urow), ur);
                    unpack8(*reinterpret_cast<const uint4*>(urow + 16), ur + 8);
                }
#pragma unroll
                for (int it = 0; it < (C * DVT / 8) / (32 * kEpiWarps); ++it) {
                    const int idx = et + 32 * kEpiWarps * it, jg = idx / C, t = idx % C;
                    const bool in = t >= w0 && t < w1;
                    const uint4 v8 = *reinterpret_cast<const uint4*>(sm.rawv + off_raw(t, jg));
                    const uint4 b8 = *reinterpret_cast<const uint4*>(sm.rawv + VB * kBox + off_raw(t, jg));
                    uint4 o8 = make_uint4(0u, 0u, 0u, 0u);
                    if constexpr (PRE) {
                        float vf[8], bf8[8], of[8];
                        unpack8(v8, vf);
                        if constexpr (LR) {
                            // pre-activation u_t . w_up[:, jg*8 + e] (the warp reads
                            // one w row: a shared-memory broadcast)
                            const float4* w4 = reinterpret_cast<const float4*>(
                                sm.rawv + VB * kBox + kLrTileBytes) + jg * 2;
#pragma unroll
                            for (int e = 0; e < 8; ++e) bf8[e] = 0.0f;
#pragma unroll
                            for (int rho = 0; rho < kLrMax; ++rho) {
                                const float4 wa = w4[rho * (DVT / 4)], wb = w4[rho * (DVT / 4) + 1];
                                bf8[0] = fmaf(ur[rho], wa.x, bf8[0]); bf8[1] = fmaf(ur[rho], wa.y, bf8[1]);
                                bf8[2] = fmaf(ur[rho], wa.z, bf8[2]); bf8[3] = fmaf(ur[rho], wa.w, bf8[3]);
                                bf8[4] = fmaf(ur[rho], wb.x, bf8[4]); bf8[5] = fmaf(ur[rho], wb.y, bf8[5]);
                                bf8[6] = fmaf(ur[rho], wb.z, bf8[6]); bf8[7] = fmaf(ur[rho], wb.w, bf8[7]);
                            }
                        } else {
                            unpack8(b8, bf8);
                        }
                        activate_beta8(bf8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) of[e] = vf[e] * bf8[e];
                        if (in) o8 = pack8(of);
                    } else {
                        if (in) o8 = bmul8(v8, b8);
                    }
                    *reinterpret_cast<uint4*>(sm.vh[ob] + off_vh(t, jg * 8)) = o8;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sm.vh_full[ob]);
                    if (w1 == nval) mbar_arrive(&sm.v_empty);  // last window of the chunk
                }
            }
            if (!p2) {
                // state-only pass: nothing to read until the last chunk of a piece,
                // after which dS holds its S_loc and the slot its log2 D; after the
                // CTA's last piece (chunk a0), the entry state of its segment
                if (p1last) {
                    const float ld2 = sm.gm[ob][iS];
                    if (!mbar_wait_own(&sm.mma1_done, nm1 & 1, fail, WL)) break;
                    ++nm1;
                    tc_fence_after();
                    ld_cols(K::COL_S, S, true);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&sm.as_free);
                        mbar_arrive(&sm.ops_empty[ob]);
                    }
                    if (!publish_piece(2 * seg + ((split1 && c == g1.mid) ? 1 : 0), ld2)) break;
                    if (c == g1.a0 && !fold_earlier()) break;
                } else {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.ops_empty[ob]);
                }
                ++item;
                continue;
            }
            if (!mbar_wait_own(&sm.mma1_done, nm1 & 1, fail, WL)) break;
            ++nm1;
            tc_fence_after();
            // saved states: the state in force before every chunk of the size asked
            // for, i.e. before window starts that are multiples of it
            const bool save_here = p.saved != nullptr && (w0 % p.chunk) == 0;
            const int cs = (c * C + w0) / p.chunk;
            {
                // A -> causal mask -> bf16 operand (row t = tA, columns s = a0 + e)
                {
                    const int a0 = 32 * hf + 16 * eh;
                    float v[16];
                    tmem_ld16_split<32>(tmem + lb + K::COL_A + 16 * eh, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = (a0 + e <= tA) ? v[e] : 0.0f;
#pragma unroll
                    for (int s8 = 0; s8 < 2; ++s8)
                        *reinterpret_cast<uint4*>(sm.abf + off_rowmajor64(tA, a0 + 8 * s8)) =
                            pack8(v + 8 * s8);
                }
                // S_hat = diag(exp(m)) S_prev, and the chunk-start state if requested
                {
                    const float em = sm.em[ob][iS];
#pragma unroll
                    for (int jg = 0; jg < SC / 8; ++jg) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = S[jg * 8 + e] * em;
                        *reinterpret_cast<uint4*>(sm.shat + off_shat<DK>(iS, sc0 + jg * 8)) = pack8(x);
                    }
                    if constexpr (!K::STAGE_SAVED) {
                        if (save_here) {
                            float4* dst = reinterpret_cast<float4*>(
                                p.saved + (((size_t)bh * NCS + cs) * DK + iS) * p.dv + j0 + sc0);
#pragma unroll
                            for (int j4 = 0; j4 < SC / 4; ++j4)
                                dst[j4] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.abf_full);
                if constexpr (K::STAGE_SAVED) {
                    // the chunk-start state (S still holds it until the update below)
                    if (save_here) {
                        if (threadIdx.x == 0) bulk_wait_read_all();  // previous store has read sstage
                        epi_sync();
#pragma unroll
                        for (int j4 = 0; j4 < SC / 4; ++j4) {
                            const int col = sc0 + 4 * j4;  // 32-column boxes, 16-byte chunks
                            const uint32_t off = (uint32_t)(col >> 5) * (DK * 128) + iS * 128 +
                                                 ((((col & 31) >> 2) ^ (iS & 7)) << 4);
                            *reinterpret_cast<float4*>(sm.sstage + off) =
                                make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
                        }
                        fence_proxy_async_smem();
                        epi_sync();
                        if (threadIdx.x == 0) {
#pragma unroll
                            for (int bx = 0; bx < DVT / 32; ++bx)
                                tma_store_2d(&A.msv, sm.sstage + bx * (DK * 128), j0 + 32 * bx,
                                             (int)(((size_t)bh * NCS + cs) * DK));
                            bulk_commit();
                        }
                    }
                }
            }
            // state update S = diag(gamma) S + diag(cfac) (Kt^T Vh)
            {
                const float gmv = sm.gm[ob][iS], cfv = sm.cf[ob][iS];
                float v[SC];
                ld_cols(K::COL_S, v, true);
#pragma unroll
                for (int e = 0; e < SC; ++e) S[e] = fmaf(gmv, S[e], cfv * v[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.as_free);
            // the constants of this item are consumed: its operand slot can refill
            // once the tensor core is done with it too
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.ops_empty[ob]);
            // o of the previous o-item (its MMA finished while this item's A and
            // state were processed), then of this one if it is the last
            if (io > 0 && !store_o(io - 1, pc, pw0, pw1)) break;
            if (last) {
                store_o(io, c, w0, w1);
                break;
            }
            pc = c;
            pw0 = w0;
            pw1 = w1;
            ++io;
            ++item;
        }
        if (threadIdx.x == 0) bulk_wait_all();  // the o stores have landed
        if (!*fail && p.ST && seg == P - 1) {
            float4* dst = reinterpret_cast<float4*>(p.ST + ((size_t)bh * DK + iS) * p.dv + j0 + sc0);
#pragma unroll
            for (int j4 = 0; j4 < SC / 4; ++j4)
                dst[j4] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, K::TMEM_COLS);
    }
    if (threadIdx.x == 0 && sm.fail) atomicOr(p.err, kErrTimeout);
}

// ------------------------------------------------------------------ host side

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct SegPlan {
    int DVT, P;
    size_t st_bytes, ld_bytes, flag_bytes, total;
};

SegPlan make_plan(const SeqParams& p, int DVT, int P) {
    const long long units = (long long)p.B * p.H * (p.dv / DVT);
    SegPlan s;
    s.DVT = DVT;
    s.P = P;
    // two piece slots per segment
    s.st_bytes = align256((size_t)2 * P * units * p.dk * DVT * 4);
    s.ld_bytes = align256((size_t)2 * P * units * p.dk * 4);
    s.flag_bytes = align256((size_t)2 * P * units * 4);
    s.total = P > 1 ? s.st_bytes + s.ld_bytes + s.flag_bytes : 0;
    return s;
}

// Slice width and segment count.  Per CTA, a chunk costs about 1 time unit
// with 64 d_v columns and 1.6 with 128 (the gate work is shared by the
// columns), and a segmented CTA spends about 0.6 more per chunk on its share
// of the state-only work.  Segments: as many as fill the SMs with one CTA
// each, none shorter than kMinSegChunks chunks, and no state-only range cut
// twice.  Take the cheaper of the two widths (128 only exists for d_k = 64,
// d_v = 128); `allow_seg` false forces P = 1.
SegPlan choose_plan(const SeqParams& p, bool allow_seg) {
    const int NC = (p.T + C - 1) / C;
    const int nsm = sm_count();
    SegPlan best{};
    double best_cost = 0.0;
    for (int DVT : {64, 128}) {
        if (DVT == 128 && !(p.dk == 64 && p.dv == 128)) continue;
        if (p.dv % DVT) continue;
        const long long units = (long long)p.B * p.H * (p.dv / DVT);
        long long P = 1;
        if (allow_seg && units < nsm) P = nsm / units;
        if (P > NC / kMinSegChunks) P = NC / kMinSegChunks;
        if (P > kMaxSeg) P = kMaxSeg;
        while (P > 1 && !p1_ranges_ok(NC, (int)P)) --P;
        if (P < 1) P = 1;
        const long long waves = (units * P + nsm - 1) / nsm;
        const double per_chunk = (DVT == 128 ? 1.6 : 1.0) * (P > 1 ? 1.6 : 1.0);
        const double cost = (double)waves * ((NC + P - 1) / P) * per_chunk;
        if (best.P == 0 || cost < best_cost) {
            best = make_plan(p, DVT, (int)P);
            best_cost = cost;
        }
    }
    return best;
}

template <int DK, int DVT, bool PRE, bool FEED, bool LR>
cudaError_t launch_cfg(const SeqParams& p, SegPlan plan, cudaStream_t s) {
    FwdKernelArgs a;
    a.p = p;
    const uint64_t BH = (uint64_t)p.B * p.H;
    if (!make_tmap_bf16_3d(&a.mq, p.q, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mk, p.k, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mg, p.g, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mt, p.tau, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mv, p.v, p.dv, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mo, p.o, p.dv, p.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    if (LR ? !make_tmap_bf16_3d_plain(&a.mu, p.beta_u, p.beta_rank, p.T, p.B, kLrMax, 64)
           : !make_tmap_bf16_3d(&a.mb, p.beta, p.dv, p.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    if (Cfg<DK, DVT>::STAGE_SAVED && p.saved &&
        !make_tmap_f32_2d(&a.msv, p.saved, p.dv, BH * (uint64_t)((p.T + p.chunk - 1) / p.chunk) * DK,
                          32, DK))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(FwdSmem<DK, DVT>) + 1024;
    auto kern = tc_fwd_kernel<DK, DVT, PRE, FEED, LR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned units = (unsigned)(BH * (p.dv / DVT));
    uint8_t* ws = static_cast<uint8_t*>(p.ws);
    a.seg.P = plan.P;
    a.seg.epoch = next_launch_tag();
    a.seg.st = plan.P > 1 ? reinterpret_cast<float*>(ws) : nullptr;
    a.seg.ld = plan.P > 1 ? reinterpret_cast<float*>(ws + plan.st_bytes) : nullptr;
    a.seg.flag = plan.P > 1 ? reinterpret_cast<unsigned*>(ws + plan.st_bytes + plan.ld_bytes) : nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * (unsigned)plan.P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;  // segments wait on one another
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = plan.P > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool PRE, bool FEED, bool LR>
cudaError_t launch_plan_t(const SeqParams& p, const SegPlan& plan, cudaStream_t s) {
    if (p.dk == 128) return launch_cfg<128, 64, PRE, FEED, LR>(p, plan, s);
    return plan.DVT == 128 ? launch_cfg<64, 128, PRE, FEED, LR>(p, plan, s)
                           : launch_cfg<64, 64, PRE, FEED, LR>(p, plan, s);
}

template <bool FEED>
cudaError_t launch_plan_f(const SeqParams& p, const SegPlan& plan, cudaStream_t s) {
    if (p.beta_rank > 0) return launch_plan_t<true, FEED, true>(p, plan, s);  // implies preact
    return p.preact ? launch_plan_t<true, FEED, false>(p, plan, s)
                    : launch_plan_t<false, FEED, false>(p, plan, s);
}

cudaError_t launch_plan(const SeqParams& p, const SegPlan& plan, cudaStream_t s) {
    return p.dfeed ? launch_plan_f<true>(p, plan, s) : launch_plan_f<false>(p, plan, s);
}

}  // namespace

bool tc_fwd_supported(const SeqParams& p) {
    return p.bf16 && (p.chunk == 16 || p.chunk == 32 || p.chunk == C) && p.T >= 1 &&
           (p.dk == 64 || p.dk == 128) &&
           (p.dv == 64 || p.dv == 128);
}

size_t tc_fwd_workspace(const SeqParams& p) {
    if (!tc_fwd_supported(p)) return 0;
    return choose_plan(p, true).total;
}

cudaError_t launch_tc_fwd(const SeqParams& p, cudaStream_t s) {
    if (!tc_fwd_supported(p)) return cudaErrorNotSupported;
    SegPlan plan = choose_plan(p, true);
    if (plan.P > 1 && (p.ws == nullptr || p.ws_bytes < plan.total)) plan = choose_plan(p, false);
    cudaError_t e = launch_plan(p, plan, s);
    if (e == cudaErrorCooperativeLaunchTooLarge && plan.P > 1) {
        (void)cudaGetLastError();  // the CTAs do not all fit at once: run unsegmented
        e = launch_plan(p, choose_plan(p, false), s);
    }
    return e;
}

}  // namespace rdm
