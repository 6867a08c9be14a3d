// tc_fwd.cu -- chunkwise-parallel DDTS forward on the sm_100a tensor cores.
//
// Rodimus trains the DDTS recurrence chunk by chunk (paperhub.cn rebuttal,
// answer to Q2 and "Efficient Parallelization": selection only along d_k makes
// the chunkwise form possible).  Per (b,h) and chunk of C = 64 tokens, with
// b_t the inclusive running sum of log(alpha) = -g*tau inside the window and
// m a per-channel reference (the midpoint of the window's b range):
//
//   Qt = q * exp(b_t - m)              Kt = k * alpha_hat * exp(m - b_s)
//   A  = mask_{s<=t}(Qt Kt^T)          Vh = beta_hat * v
//   o  = A Vh + Qt (diag(exp(m)) S_prev)                 (intra + inter chunk)
//   S  = diag(exp(b_last)) S_prev + diag(exp(b_last - m)) Kt^T Vh
//
// Every factor stays inside exp(+-span/2) with span = b_first - b_last of the
// window, so products are exact in fp32 range whenever span <= kSpanMax.  A
// chunk whose span is larger is processed as windows of 16 tokens, or of 1
// token, each window being one pass of the same pipeline (exact for any decay).
//
// One CTA owns one (b,h) and a 64-wide slice of d_v.  Warp roles:
//   warps 0-3  epilogue: A -> masked bf16 operand, state (fp32 registers),
//              S_hat operand, o store (TMEM lanes = rows)
//   warps 4-7  gates: TMA tiles -> log-decay scan, Qt, Kt, Vh operands (bf16)
//   warp  8    TMA producer (q, k, g, tau, v, beta tiles, 128B-swizzled)
//   warp  9    TMEM allocator and single-thread tcgen05.mma issuer
// All hand-offs are mbarriers with bounded waits (a timeout sets the device
// status word and the CTA exits cleanly).
#include <cuda.h>

#include "launch.h"
#include "rdm_common.cuh"
#include "tc_common.cuh"

namespace rdm {
namespace {
using namespace tc;

constexpr int C = 64;                        // tokens per chunk (tile rows)
constexpr int kGateWarps = 8;  // two per SM sub-partition
constexpr int kThreads = 32 * (4 + kGateWarps + 2);
constexpr int kEpiWarp0 = 0, kGateWarp0 = 4, kProdWarp = 4 + kGateWarps, kMmaWarp = 5 + kGateWarps;
constexpr int kBarGate = 3;  // all gate warps

template <int DK, int DVT>
struct Cfg {
    static constexpr int NS = DK == 128 ? 1 : 2;   // raw TMA stages
    static constexpr int NB = 2;                   // operand buffers
    static constexpr int KB = DK / 64;             // boxes per key-side tile
    static constexpr int VB = DVT / 64;            // boxes per value-side tile
    static constexpr int RAW = (4 * KB + 2 * VB) * kBox;
    static constexpr int G = DK / 8;               // 8-channel groups
    // A | dS | O (double-buffered: the epilogue reads O of one chunk while the
    // tensor core writes the next)
    static constexpr int COL_A = 0, COL_S = 64, COL_O = 64 + DVT;
    static constexpr int TMEM_COLS = (64 + 3 * DVT) <= 256 ? 256 : 512;
};

template <int DK, int DVT>
struct alignas(1024) FwdSmem {
    using K = Cfg<DK, DVT>;
    uint8_t raw[K::NS][K::RAW];
    uint8_t qt[K::NB][K::G * kQK];
    uint8_t kt[K::NB][K::G * kQK];
    uint8_t vh[K::NB][C * DVT * 2];
    uint8_t abf[C * C * 2];
    uint8_t shat[DK * DVT * 2];
    float em[K::NB][DK], cf[K::NB][DK], gm[K::NB][DK];
    int info[K::NB][4];  // chunk, w0, w1, last
    uint64_t raw_full[K::NS], raw_empty[K::NS], ops_full[K::NB], ops_empty[K::NB];
    uint64_t mma1_done, as_free, abf_full, mmao_done[2], o_free[2];
    int need16[2], need1[2];
    uint32_t tmem_base;
    int fail;
};

struct FwdKernelArgs {
    CUtensorMap mq, mk, mg, mt, mv, mb;
    SeqParams p;
};

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads, 1) tc_fwd_kernel(const __grid_constant__ FwdKernelArgs A) {
    using K = Cfg<DK, DVT>;
    constexpr int NS = K::NS, NB = K::NB, KB = K::KB, VB = K::VB;
    // align by pointer arithmetic on the __shared__ array so that every access
    // below stays a shared-memory access (an integer round trip would make it generic)
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    FwdSmem<DK, DVT>& sm = *reinterpret_cast<FwdSmem<DK, DVT>*>(
        smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
    const SeqParams& p = A.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NJ = p.dv / DVT;
    const int bh = blockIdx.x / NJ, j0 = (blockIdx.x % NJ) * DVT;
    const int T = p.T, NC = (T + C - 1) / C;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.raw_full[s], 1);
            mbar_init(&sm.raw_empty[s], kGateWarps);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&sm.ops_full[b], kGateWarps);
            mbar_init(&sm.ops_empty[b], 1 + 4);
        }
        mbar_init(&sm.mma1_done, 1);
        mbar_init(&sm.as_free, 4);
        mbar_init(&sm.abf_full, 4);
        mbar_init(&sm.mmao_done[0], 1);
        mbar_init(&sm.mmao_done[1], 1);
        mbar_init(&sm.o_free[0], 4);
        mbar_init(&sm.o_free[1], 4);
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
        prefetch_tmap(&A.mt); prefetch_tmap(&A.mv); prefetch_tmap(&A.mb);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* fail = &sm.fail;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < NC; ++c) {
                const int st = c % NS;
                if (c >= NS && !mbar_wait(&sm.raw_empty[st], ((c / NS) - 1) & 1, fail, kWaitLimit))
                    break;
                mbar_expect_tx(&sm.raw_full[st], K::RAW);
                uint8_t* raw = sm.raw[st];
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_3d(raw + (0 * KB + kb) * kBox, &A.mq, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (1 * KB + kb) * kBox, &A.mk, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (2 * KB + kb) * kBox, &A.mg, &sm.raw_full[st], 64 * kb, c * C, bh);
                    tma_load_3d(raw + (3 * KB + kb) * kBox, &A.mt, &sm.raw_full[st], 64 * kb, c * C, bh);
                }
                for (int vb = 0; vb < VB; ++vb) {
                    tma_load_3d(raw + (4 * KB + vb) * kBox, &A.mv, &sm.raw_full[st], j0 + 64 * vb, c * C, bh);
                    tma_load_3d(raw + (4 * KB + VB + vb) * kBox, &A.mb, &sm.raw_full[st], j0 + 64 * vb, c * C, bh);
                }
                ++issued;
            }
            // never leave the CTA with copies in flight
            for (int c = issued - NS < 0 ? 0 : issued - NS; c < issued; ++c)
                drain_wait(&sm.raw_full[c % NS], (c / NS) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tA = tmem + K::COL_A, tS = tmem + K::COL_S, tO = tmem + K::COL_O;
            constexpr uint32_t id1 = idesc_bf16(64, 64, 0, 0);    // A  = Qt Kt^T
            constexpr uint32_t idS = idesc_bf16(DK, DVT, 1, 1);   // dS = Kt^T Vh
            constexpr uint32_t idO = idesc_bf16(64, DVT, 0, 1);   // O  = A Vh + Qt S_hat
            int item = 0, n1 = 0, nO = 0;
            while (true) {
                const int ob = item % NB;
                if (!mbar_wait(&sm.ops_full[ob], (item / NB) & 1, fail, kWaitLimit)) break;
                const int last = sm.info[ob][3];
                if (item > 0 && !mbar_wait(&sm.as_free, (item - 1) & 1, fail, kWaitLimit)) break;
                tc_fence_after();
                const uint32_t q = smem_u32(sm.qt[ob]), k = smem_u32(sm.kt[ob]);
                const uint32_t v = smem_u32(sm.vh[ob]);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    mma_bf16(tA, sdesc(q + ks * 2 * kQK, kQK, 128), sdesc(k + ks * 2 * kQK, kQK, 128),
                             id1, ks > 0);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tS, sdesc(k + ks * 256, 128, kQK), sdesc(v + ks * 256, 128, 1024), idS,
                             ks > 0);
                mma_commit(&sm.mma1_done);
                ++n1;
                if (!mbar_wait(&sm.abf_full, item & 1, fail, kWaitLimit)) break;
                const int obuf = item & 1;
                if (item >= 2 && !mbar_wait(&sm.o_free[obuf], ((item >> 1) - 1) & 1, fail, kWaitLimit)) break;
                tc_fence_after();
                const uint32_t a = smem_u32(sm.abf), sh = smem_u32(sm.shat);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tO + obuf * DVT, sdesc(a + ks * 2048, 1024, 128),
                             sdesc(v + ks * 256, 128, 1024), idO, ks > 0);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    mma_bf16(tO + obuf * DVT, sdesc(q + ks * 2 * kQK, kQK, 128),
                             sdesc(sh + ks * 256, 128, DK * 16), idO, 1);
                mma_commit(&sm.mmao_done[obuf]);
                mma_commit(&sm.ops_empty[ob]);
                ++nO;
                if (last) break;
                ++item;
            }
            // let issued MMAs finish before TMEM is released
            if (n1 > 0) drain_wait(&sm.mma1_done, (n1 - 1) & 1);
            if (nO > 0) drain_wait(&sm.mmao_done[(nO - 1) & 1], ((nO - 1) >> 1) & 1);
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
        const int cgl = lane % GW, seg = lane / GW;
        const int cg = gw * GW + cgl;
        const int tb = seg * SEGT;  // first token of my segment
        const uint32_t full = 0xffffffffu;
        int item = 0;
        for (int c = 0; c < NC; ++c) {
            const int st = c % NS;
            if (!mbar_wait(&sm.raw_full[st], (c / NS) & 1, fail, kWaitLimit)) break;
            const uint8_t* raw = sm.raw[st];
            const int nval = min(C, T - c * C);
            float b[SEGT][8], bf[8], bl[8];
            // window-relative inclusive running sum of log(alpha) over my tokens, and
            // b at the first / last valid token of my window (W in {64, 16})
            auto scan = [&](int W) {
#pragma unroll
                for (int u = 0; u < SEGT; ++u) {
                    float g8[8], t8[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(tb + u, cg)), g8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(tb + u, cg)), t8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float la = (tb + u < nval) ? log_alpha(g8[e], t8[e]) : 0.0f;
                        b[u][e] = (u == 0 || W == 1) ? la : b[u - 1][e] + la;
                    }
                }
                if (W == 1) return;
                const int WL = W / SEGT * GW;        // lanes per window
                const int l0 = lane & ~(WL - 1);     // first lane of my window
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
                        if ((lane & (WL - 1)) >= d) x += y;
                    }
                    const float excl = x - tot;
                    float mine = 0.0f;
#pragma unroll
                    for (int u = 0; u < SEGT; ++u) {
                        b[u][e] += excl;
                        if (u == usrc) mine = b[u][e];
                    }
                    bf[e] = __shfl_sync(full, b[0][e], l0 + cgl);
                    bl[e] = __shfl_sync(full, mine, lsrc);
                }
            };
            // true when some window of this chunk spans more log-decay than one
            // reference holds; every gate warp takes the same answer
            auto too_wide = [&](int* flag) {
                float span = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) span = fmaxf(span, bf[e] - bl[e]);
                if (tb >= nval) span = 0.0f;
                if (__any_sync(full, !(span <= kSpanMax)) && lane == 0) *flag = c + 1;
                named_bar(kBarGate, 32 * kGateWarps);
                return *flag == c + 1;
            };
            int W = C;
            scan(C);
            if (too_wide(&sm.need16[c & 1])) {
                W = 16;
                scan(16);
                if (too_wide(&sm.need1[c & 1])) {
                    W = 1;
                    scan(1);
                }
            }
            // Vh = beta_hat * v for the rows of [w0, w1), zero elsewhere
            auto write_vh = [&](int ob, int w0, int w1) {
#pragma unroll
                for (int it = 0; it < VIT; ++it) {
                    const int jg = gt / TPG, t = (gt % TPG) + TPG * it;
                    const bool in = t >= w0 && t < w1;
                    float v8[8], b8[8], o8[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 4 * KB * kBox + off_raw(t, jg)), v8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + (4 * KB + VB) * kBox + off_raw(t, jg)), b8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o8[e] = in ? v8[e] * b8[e] : 0.0f;
                    *reinterpret_cast<uint4*>(sm.vh[ob] + off_vh(t, jg * 8)) = pack8(o8);
                }
            };
            auto publish = [&](int ob, int w0, int w1) {
                if (gt == 0) {
                    sm.info[ob][0] = c;
                    sm.info[ob][1] = w0;
                    sm.info[ob][2] = w1;
                    sm.info[ob][3] = (c == NC - 1) && (w1 == nval);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.ops_full[ob]);
            };
            if (W == C) {
                // ---- one window = the whole chunk (rows past T hold zeros from the
                // TMA fill, so every row can be computed unmasked)
                const int ob = item % NB;
                if (item >= NB && !mbar_wait(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, kWaitLimit))
                    break;
                float mL[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mL[e] = 0.5f * (bf[e] + bl[e]) * kLog2e;
#pragma unroll
                for (int u = 0; u < SEGT; ++u) {
                    const int t = tb + u;
                    float q8[8], k8[8], g8[8], t8[8], oq[8], ok[8];
                    unpack8(*reinterpret_cast<const uint4*>(raw + 0 * KB * kBox + off_raw(t, cg)), q8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + 1 * KB * kBox + off_raw(t, cg)), k8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + 2 * KB * kBox + off_raw(t, cg)), g8);
                    unpack8(*reinterpret_cast<const uint4*>(raw + 3 * KB * kBox + off_raw(t, cg)), t8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float d = fmaf(b[u][e], kLog2e, -mL[e]);
                        const float lah = t8[e] == 0.0f ? 0.0f : t8[e] * lg2_fast(g8[e]);
                        oq[e] = q8[e] * ex2_fast(d);
                        ok[e] = k8[e] * ex2_fast(lah - d);
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
                publish(ob, 0, nval);
                ++item;
            } else {
                bool ok_loop = true;
                for (int w0 = 0; w0 < nval; w0 += W) {
                    const int w1 = min(w0 + W, nval);
                    const int ob = item % NB;
                    if (item >= NB &&
                        !mbar_wait(&sm.ops_empty[ob], ((item / NB) - 1) & 1, fail, kWaitLimit)) {
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
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            // reference m = midpoint of the window's b range, blast = b at its end
                            const float blast = W == 1 ? b[u][e] : bl[e];
                            const float m = W == 1 ? b[u][e] : 0.5f * (bf[e] + bl[e]);
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
                    publish(ob, w0, w1);
                    ++item;
                }
                if (!ok_loop) break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.raw_empty[st]);
            if (*fail) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;
        const bool rowA = lane < 16;                      // valid rows of A and O (M = 64)
        const int tA = 16 * ew + lane;
        const bool rowS = (DK == 128) || lane < 16;        // valid state rows (M = DK)
        const int iS = (DK == 128) ? 32 * ew + lane : 16 * ew + lane;
        const uint32_t lb = (uint32_t)(32 * ew) << 16;
        float S[DVT];
#pragma unroll
        for (int j = 0; j < DVT; ++j)
            S[j] = (rowS && p.S0) ? p.S0[((size_t)bh * DK + iS) * p.dv + j0 + j] : 0.0f;
        // o rows [w0, w1) of chunk c from the O buffer of item `it`
        auto store_o = [&](int it, int c, int w0, int w1) -> bool {
            const int obuf = it & 1;
            if (!mbar_wait(&sm.mmao_done[obuf], (it >> 1) & 1, fail, kWaitLimit)) return false;
            tc_fence_after();
            const bool st_row = rowA && tA >= w0 && tA < w1;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) +
                                  ((size_t)bh * T + (size_t)c * C + tA) * p.dv + j0;
#pragma unroll
            for (int qd = 0; qd < DVT / 32; ++qd) {
                float v[32];
                tmem_ld32(tmem + lb + K::COL_O + obuf * DVT + 32 * qd, v);
                tmem_ld_wait();
                if (st_row) {
#pragma unroll
                    for (int sg = 0; sg < 4; ++sg)
                        reinterpret_cast<uint4*>(orow)[4 * qd + sg] = pack8(v + 8 * sg);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.o_free[obuf]);
            return true;
        };
        int item = 0, pc = 0, pw0 = 0, pw1 = 0;
        while (true) {
            const int ob = item % NB;
            if (!mbar_wait(&sm.ops_full[ob], (item / NB) & 1, fail, kWaitLimit)) break;
            const int c = sm.info[ob][0], w0 = sm.info[ob][1], w1 = sm.info[ob][2];
            const int last = sm.info[ob][3];
            if (!mbar_wait(&sm.mma1_done, item & 1, fail, kWaitLimit)) break;
            tc_fence_after();
            // A -> causal mask -> bf16 operand (row t = tA, columns s)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float v[32];
                tmem_ld32(tmem + lb + K::COL_A + 32 * hf, v);
                tmem_ld_wait();
                if (rowA) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = (32 * hf + e <= tA) ? v[e] : 0.0f;
#pragma unroll
                    for (int sg = 0; sg < 4; ++sg)
                        *reinterpret_cast<uint4*>(sm.abf + off_rowmajor64(tA, 32 * hf + 8 * sg)) =
                            pack8(v + 8 * sg);
                }
            }
            // S_hat = diag(exp(m)) S_prev, and the chunk-start state if requested
            if (rowS) {
                const float em = sm.em[ob][iS];
#pragma unroll
                for (int jg = 0; jg < DVT / 8; ++jg) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = S[jg * 8 + e] * em;
                    *reinterpret_cast<uint4*>(sm.shat + off_shat<DK>(iS, jg * 8)) = pack8(x);
                }
                if (p.saved && w0 == 0) {
                    float4* dst = reinterpret_cast<float4*>(
                        p.saved + (((size_t)bh * NC + c) * DK + iS) * p.dv + j0);
#pragma unroll
                    for (int j4 = 0; j4 < DVT / 4; ++j4)
                        dst[j4] = make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.abf_full);
            // state update S = diag(gamma) S + diag(cfac) (Kt^T Vh)
            {
                const float gmv = rowS ? sm.gm[ob][iS] : 0.0f, cfv = rowS ? sm.cf[ob][iS] : 0.0f;
#pragma unroll
                for (int qd = 0; qd < DVT / 32; ++qd) {
                    float v[32];
                    tmem_ld32(tmem + lb + K::COL_S + 32 * qd, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) S[32 * qd + e] = fmaf(gmv, S[32 * qd + e], cfv * v[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.as_free);
            // the constants of this item are consumed: its operand slot can refill
            // once the tensor core is done with it too
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.ops_empty[ob]);
            // o of the previous item (its MMA finished while this item's A and state
            // were processed), then of this one if it is the last
            if (item > 0 && !store_o(item - 1, pc, pw0, pw1)) break;
            if (last) {
                store_o(item, c, w0, w1);
                break;
            }
            pc = c;
            pw0 = w0;
            pw1 = w1;
            ++item;
        }
        if (!*fail && rowS && p.ST) {
            float4* dst = reinterpret_cast<float4*>(p.ST + ((size_t)bh * DK + iS) * p.dv + j0);
#pragma unroll
            for (int j4 = 0; j4 < DVT / 4; ++j4)
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

template <int DK, int DVT>
cudaError_t launch_cfg(const SeqParams& p, cudaStream_t s) {
    FwdKernelArgs a;
    a.p = p;
    const uint64_t BH = (uint64_t)p.B * p.H;
    if (!make_tmap_bf16_3d(&a.mq, p.q, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mk, p.k, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mg, p.g, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mt, p.tau, p.dk, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mv, p.v, p.dv, p.T, BH, 64, 64) ||
        !make_tmap_bf16_3d(&a.mb, p.beta, p.dv, p.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(FwdSmem<DK, DVT>) + 1024;
    auto kern = tc_fwd_kernel<DK, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)(BH * (p.dv / DVT));
    kern<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool tc_fwd_supported(const SeqParams& p) {
    return p.bf16 && p.chunk == C && p.T >= 1 && (p.dk == 64 || p.dk == 128) &&
           (p.dv == 64 || p.dv == 128);
}

cudaError_t launch_tc_fwd(const SeqParams& p, cudaStream_t s) {
    if (!tc_fwd_supported(p)) return cudaErrorNotSupported;
    if (p.dk == 64) return launch_cfg<64, 64>(p, s);
    return launch_cfg<128, 64>(p, s);
}

}  // namespace rdm
