// ska.cu -- sliding-window shared-key attention (SW-SKA), the attention half of
// the Rodimus+ block ("Rodimus*: Breaking the Accuracy-Efficiency Trade-Off with
// Efficient Attentions"; digest.lyk-ai.com summary, "Method", Rodimus+ bullets:
// a sliding window for local context, one key shared by every head so the KV
// cache shrinks; paperhub.cn OpenReview rebuttal, answer to Q1: multi-head
// query and value projections, a multi-query key projection).  Per batch b,
// head h, token t:
//
//   s_u = scale * q[b,h,t] . k[b,u]   for u = max(0, t-w+1) .. t
//   o[b,h,t] = sum_u softmax(s)_u v[b,h,u]
//
// Forward (tensor cores, bf16 in, fp32 accumulation): CTAs walk tiles of 128
// queries of one (b, h) (two CTAs per SM and one tile each where TMEM allows,
// else one persistent CTA per SM); the next tile's queries load while the
// current one finishes.  TMA brings the query
// tile once and the 64-key tiles of the window through rings of four key and three value stages
// (128-byte swizzle, used by the MMA as is); tcgen05 computes S = Q K^T into
// TMEM, eight softmax warps (two per query row, each with half of the keys and
// half of the output columns) mask the window, keep the running row maximum and
// sum, write P = 2^(S*c - m) as bf16 into shared memory, and tcgen05 computes
// P V into a second TMEM buffer, which the same threads fold into registers
// with the rescale exp2(m_old - m_new).  Issue order S_n, PV_{n-1} lets the
// softmax of tile n overlap the P V product of tile n-1.
//
// Decode: one CTA per (b, group of up to eight heads) against ring caches
// (position p in slot p mod w): the new key and value are written to their slot
// and used from the inputs, each cached key row is read once for the group's
// heads, scores go through shared memory, then a coalesced sweep over the
// value rows of each head.
#include <cuda_bf16.h>
#include <stdint.h>

#include "launch.h"
#include "rdm_common.cuh"
#include "ska_launch.h"
#include "tc_common.cuh"

namespace rdm {

using namespace tc;

namespace {

constexpr int kQRows = 128;          // queries per CTA (MMA M)
// eight softmax warps: warps w and w + 4 share the TMEM lane quarter w % 4
// (query rows 32 (w % 4) ..), each taking half of the key columns of S and
// half of the output columns, so that two warps per scheduler interleave
constexpr int kSoftWarps = 8;
constexpr int kProdWarp = 8, kMmaWarp = 9;
constexpr int kSkaThreads = 320;

// Shared-memory operands: K-major 128-byte-swizzled TMA tiles (Q, K: rows of
// 64 elements in 8-row, 1024-byte atoms; descriptor layout type 2 of sm_100),
// MN-major 128-byte-swizzled V tiles (64-element rows along N), and P in the
// no-swizzle K-major layout of 8x8 core matrices.

template <int DK, int DV>
struct SkaCfg {
    static constexpr int NK = 64;  // keys per tile (MMA N of S, K of P V)
    static constexpr int Q_BYTES = kQRows * DK * 2;
    static constexpr int K_BYTES = NK * DK * 2;
    static constexpr int V_BYTES = NK * DV * 2;
    static constexpr int P_BYTES = kQRows * NK * 2;
    // S and P V double-buffered; 256 columns let two CTAs share an SM
    static constexpr uint32_t TMEM_COLS = 2 * NK + 2 * DV <= 256 ? 256 : 512;
    static constexpr int CTAS_PER_SM = TMEM_COLS == 256 && DK == 64 ? 2 : 1;
    // key and value tiles in flight (a tile takes a few microseconds to land
    // when every SM streams; keys run further ahead, the MMA waits on them first)
    static constexpr int KS = 4, VS = 3;
};

template <int DK, int DV>
struct SkaSmem {
    using K = SkaCfg<DK, DV>;
    alignas(1024) uint8_t q[K::Q_BYTES];
    alignas(1024) uint8_t k[K::KS][K::K_BYTES];
    alignas(1024) uint8_t v[K::VS][K::V_BYTES];
    alignas(1024) uint8_t p[2][K::P_BYTES];  // no-swizzle K-major (8x8 core matrices)
    uint64_t q_full, q_empty, k_full[K::KS], v_full[K::VS], k_empty[K::KS], v_empty[K::VS];
    // S, P and O buffers need no "empty" barriers: the MMA thread writes S_n and
    // O_n only after p_full of tile n-2 (resp. n), on which every softmax warp
    // arrives after it has read S_{n-2} (resp. folded O_{n-2}), and the softmax
    // writes P_n only after o_full of tile n-2 (P V of tile n-2 done)
    uint64_t s_full[2], p_full[2], o_full[2], mma_done;
    float red_max[2][2][kQRows];  // [tile parity][column half][row]: partial row maxima
    float red_sum[2][2][kQRows];  // [query-tile parity][column half][row]: partial row sums
    uint32_t tmem_base;
    int fail;
};

struct SkaKernelArgs {
    SkaParams p;
    CUtensorMap mq, mk, mv;
};

// Non-blocking probe of an mbarrier phase (test_wait returns at once; a
// try_wait would suspend the thread for a while when the phase is open, which
// would hold the producer on one ring while the other has a free stage).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Warp-uniform bounded wait of the softmax warps: every lane waits on its own
// clock (never on the shared failure flag, which another role may raise at any
// moment), then the warp agrees.  Both warps of a pair wait for the same phases
// in the same order, so they pass or run out together and never leave one
// another alone at their pair barrier; the tcgen05 loads that follow are
// warp-collective.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* fail,
                                          long long limit) {
    const bool ok = mbar_wait_own(bar, parity, fail, limit);
    return __all_sync(0xffffffffu, ok);
}

// A query tile: 128 queries of sequence bh starting at t0, and its key tiles
// j_lo .. j_lo + nt - 1 (64 keys each) covering the windows of its rows.
struct SkaTile {
    int b, bh, t0, j_lo, nt;
};
template <int NK>
__device__ __forceinline__ SkaTile ska_tile(const SkaParams& p, int g) {
    const int NQ = (p.T + kQRows - 1) / kQRows;
    SkaTile s;
    s.bh = g / NQ;
    s.b = s.bh / p.H;
    s.t0 = (g % NQ) * kQRows;
    const int lo0 = s.t0 - p.window + 1;  // first key any row of the tile can see
    s.j_lo = (lo0 > 0 ? lo0 : 0) / NK;
    s.nt = min(s.t0 + kQRows - 1, p.T - 1) / NK - s.j_lo + 1;
    return s;
}

template <int DK, int DV>
__global__ void __launch_bounds__(kSkaThreads, SkaCfg<DK, DV>::CTAS_PER_SM)
    ska_fwd_kernel(const __grid_constant__ SkaKernelArgs A) {
    using K = SkaCfg<DK, DV>;
    constexpr int NK = K::NK;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    SkaSmem<DK, DV>& sm = *reinterpret_cast<SkaSmem<DK, DV>*>(
        smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
    const SkaParams& p = A.p;
    const long long WL = p.wait_limit > 0 ? p.wait_limit : kDefaultWaitLimit;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T, NQ = (T + kQRows - 1) / kQRows;
    // persistent CTAs: query tiles g = blockIdx.x + k * gridDim.x, numbered
    // (b, h, tile) with the tiles of one sequence consecutive, so neighbouring
    // CTAs work on overlapping windows of one head at the same time (their key
    // and value tiles meet in L2)
    const int TQ = p.B * p.H * NQ;
    const int G = gridDim.x;
    const int nq = (int)blockIdx.x < TQ ? (TQ - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        for (int s = 0; s < K::KS; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < K::VS; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.p_full[s], kSoftWarps);
            mbar_init(&sm.o_full[s], 1);
        }
        mbar_init(&sm.mma_done, 1);
        sm.fail = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, K::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_tmap(&A.mq); prefetch_tmap(&A.mk); prefetch_tmap(&A.mv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tS = tmem, tO = tmem + 2 * NK;  // S buffers, then P V buffers
    volatile int* fail = &sm.fail;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        // Three independent streams, served whenever a stage is free (polled
        // with test_wait): the query tile of the next query tile (once the
        // last Q K^T of the current one has been issued and finished), key
        // tiles (a key stage frees after its Q K^T) and value tiles (a value
        // stage frees after its P V), each counted over all of the CTA's query
        // tiles in order.
        if (lane == 0 && nq > 0) {
            int qq = 0;               // query tiles whose Q has been issued
            int qk = 0, jk = 0;       // key stream: query tile, key tile within it
            int qv = p.withhold ? nq : 0, jv = 0;  // value stream (none under the test hook)
            int nk = 0, nv = 0;       // key / value tiles issued in all
            SkaTile tk = ska_tile<NK>(p, blockIdx.x), tv = tk;
            long long idle0 = clock64();
            while (qq < nq || qk < nq || qv < nq) {
                bool moved = false;
                if (qq < nq && (qq == 0 || mbar_test(&sm.q_empty, (qq - 1) & 1))) {
                    const SkaTile tq = ska_tile<NK>(p, blockIdx.x + qq * G);
                    mbar_expect_tx(&sm.q_full, K::Q_BYTES);
#pragma unroll
                    for (int x = 0; x < DK / 64; ++x)
                        tma_load_3d(sm.q + x * kQRows * 128, &A.mq, &sm.q_full, 64 * x, tq.t0, tq.bh);
                    ++qq;
                    moved = true;
                }
                if (qk < nq && mbar_test(&sm.k_empty[nk % K::KS], ((nk / K::KS) & 1) ^ 1)) {
                    const int st = nk % K::KS;
                    mbar_expect_tx(&sm.k_full[st], K::K_BYTES);
#pragma unroll
                    for (int x = 0; x < DK / 64; ++x)
                        tma_load_3d(sm.k[st] + x * NK * 128, &A.mk, &sm.k_full[st], 64 * x,
                                    (tk.j_lo + jk) * NK, tk.b);
                    ++nk;
                    if (++jk == tk.nt) {
                        jk = 0;
                        if (++qk < nq) tk = ska_tile<NK>(p, blockIdx.x + qk * G);
                    }
                    moved = true;
                }
                if (qv < nq && nv < nk && mbar_test(&sm.v_empty[nv % K::VS], ((nv / K::VS) & 1) ^ 1)) {
                    const int st = nv % K::VS;
                    mbar_expect_tx(&sm.v_full[st], K::V_BYTES);
#pragma unroll
                    for (int x = 0; x < DV / 64; ++x)
                        tma_load_3d(sm.v[st] + x * NK * 128, &A.mv, &sm.v_full[st], 64 * x,
                                    (tv.j_lo + jv) * NK, tv.bh);
                    ++nv;
                    if (++jv == tv.nt) {
                        jv = 0;
                        if (++qv < nq) tv = ska_tile<NK>(p, blockIdx.x + qv * G);
                    }
                    moved = true;
                }
                if (moved) {
                    idle0 = clock64();
                } else if (*fail) {
                    break;
                } else if (clock64() - idle0 > WL) {
                    *fail = 1;
                    break;
                }
            }
            // no copy may land after the CTA has gone: wait (bounded, on our own
            // clock) for the last ones issued into each stage and for the query
            if (qq > 0) mbar_wait_own(&sm.q_full, (qq - 1) & 1, fail, WL);
            for (int n = nk - K::KS > 0 ? nk - K::KS : 0; n < nk; ++n)
                mbar_wait_own(&sm.k_full[n % K::KS], (n / K::KS) & 1, fail, WL);
            for (int n = nv - K::VS > 0 ? nv - K::VS : 0; n < nv; ++n)
                mbar_wait_own(&sm.v_full[n % K::VS], (n / K::VS) & 1, fail, WL);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(kQRows, NK, 0, 0);  // S = Q K^T
            constexpr uint32_t idO = idesc_bf16(kQRows, DV, 0, 1);  // O = P V (V MN-major)
            // Descriptors as two 32-bit words, built once: the low word is the
            // start address / 16 plus the leading offset, so the operand of step
            // ks of stage s is base + a constant (one add per MMA); the high word
            // (stride offset, sm_100 version bit, layout) is fixed per operand.
            constexpr uint32_t kSw128 = 2u << 29;
            const uint32_t q_lo = (smem_u32(sm.q) >> 4) | (1u << 16);
            const uint32_t k_lo = (smem_u32(sm.k[0]) >> 4) | (1u << 16);
            const uint32_t p_lo = (smem_u32(sm.p[0]) >> 4) | ((128u >> 4) << 16);
            const uint32_t v_lo = (smem_u32(sm.v[0]) >> 4) | (((uint32_t)NK * 128 >> 4) << 16);
            constexpr uint32_t qk_hi = (1024u >> 4) | (1u << 14) | kSw128;
            constexpr uint32_t p_hi = ((uint32_t)NK * 16 >> 4) | (1u << 14);
            constexpr uint32_t v_hi = (1024u >> 4) | (1u << 14) | kSw128;
            auto pv = [&](int m) -> bool {
                const int st = m & 1, vs = m % K::VS;
                const uint32_t ph = (m >> 1) & 1;
                // p_full[m] also means the softmax has read O_{m-2} out of buffer
                // st (each warp folds tile m-2 before it writes P_m)
                if (!mbar_wait(&sm.p_full[st], ph, fail, WL)) return false;
                if (!mbar_wait(&sm.v_full[vs], (m / K::VS) & 1, fail, WL)) return false;
                tc_fence_after();
                const uint32_t pa = p_lo + st * (K::P_BYTES >> 4), va = v_lo + vs * (K::V_BYTES >> 4);
#pragma unroll
                for (int ks = 0; ks < NK / 16; ++ks)
                    mma_bf16_w(tO + st * DV, pa + ks * (256 >> 4), p_hi, va + ks * (2048 >> 4), v_hi, idO,
                               ks > 0);
                mma_commit(&sm.o_full[st]);  // also frees P buffer st for P_{m+2}
                mma_commit(&sm.v_empty[vs]);
                return true;
            };
            // Per key tile n (counted over all query tiles): S_n, then P V of
            // the previous key tile of the same query tile; the last key tile of
            // a query tile has its P V issued right after its S, so that the
            // softmax can finish the query tile while the next one's query is
            // loaded.  P V of tile m is therefore issued before S_{m+2}: S and O
            // buffers are free by the p_full argument above.
            bool ok = true;
            int n = 0;
            for (int qi = 0; ok && qi < nq; ++qi) {
                const SkaTile tq = ska_tile<NK>(p, blockIdx.x + qi * G);
                if (!mbar_wait(&sm.q_full, qi & 1, fail, WL)) { ok = false; break; }
                for (int j = 0; j < tq.nt; ++j, ++n) {
                    const int st = n & 1, ks_ = n % K::KS;
                    if (!mbar_wait(&sm.k_full[ks_], (n / K::KS) & 1, fail, WL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t ka = k_lo + ks_ * (K::K_BYTES >> 4);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks) {
                        const uint32_t off = ((ks / 4) * (kQRows * 128) + (ks % 4) * 32) >> 4;
                        const uint32_t koff = ((ks / 4) * (NK * 128) + (ks % 4) * 32) >> 4;
                        mma_bf16_w(tS + st * NK, q_lo + off, qk_hi, ka + koff, qk_hi, idS, ks > 0);
                    }
                    mma_commit(&sm.s_full[st]);
                    mma_commit(&sm.k_empty[ks_]);
                    const bool last = j == tq.nt - 1;
                    if (last) mma_commit(&sm.q_empty);  // the query tile may be replaced
                    if (j > 0 && !(ok = pv(n - 1))) break;
                    if (last && !(ok = pv(n))) break;
                }
            }
            // every MMA issued has finished before TMEM is released
            mma_commit(&sm.mma_done);
            mbar_wait_own(&sm.mma_done, 0, fail, WL);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------- softmax
        constexpr int NH = NK / 2, DH = DV / 2;  // key / output columns of this warp
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;  // query row = TMEM lane
        const float c = p.scale * kLog2e;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int bar_pair = 1 + quarter;  // named barrier of warps quarter, quarter + 4
        float o[DH];
        float m_run, l, corr_pending;
        auto fold = [&](int i, float cr) -> bool {
            const int st = i & 1;
            if (!warp_wait(&sm.o_full[st], (i >> 1) & 1, fail, WL)) return false;
            tc_fence_after();
            float x[DH];
#pragma unroll
            for (int q32 = 0; q32 < DH / 32; ++q32)
                tmem_ld32(tO + st * DV + half * DH + lane_off + q32 * 32, x + q32 * 32);
            tmem_ld_wait();
            tc_fence_before();  // ordered before the next p_full arrival
#pragma unroll
            for (int j = 0; j < DH; ++j) o[j] = fmaf(o[j], cr, x[j]);
            return true;
        };
        bool ok = true;
        int n = 0;  // key tile, counted over all query tiles
        for (int qi = 0; ok && qi < nq; ++qi) {
            const SkaTile tq = ska_tile<NK>(p, blockIdx.x + qi * G);
            const int t = tq.t0 + r;
            const int lo = t - p.window + 1, hi = min(t, T - 1);
#pragma unroll
            for (int j = 0; j < DH; ++j) o[j] = 0.0f;
            m_run = -INFINITY;
            l = 0.0f;
            corr_pending = 1.0f;
            for (int j = 0; j < tq.nt; ++j, ++n) {
                const int st = n & 1;
                const uint32_t ph = (n >> 1) & 1;
                // the pair's warps meet at bar_pair below: both reach it or, after a
                // failed wait, neither does (the waits are warp-uniform and both warps
                // of a pair wait for the same phases)
                if (!warp_wait(&sm.s_full[st], ph, fail, WL)) { ok = false; break; }
                tc_fence_after();
                float s_[NH];
#pragma unroll
                for (int q32 = 0; q32 < NH / 32; ++q32)
                    tmem_ld32(tS + st * NK + half * NH + lane_off + q32 * 32, s_ + q32 * 32);
                tmem_ld_wait();
                tc_fence_before();  // ordered before this tile's p_full arrival
                const int kb = (tq.j_lo + j) * NK + half * NH;
                if (kb < lo || kb + NH - 1 > hi) {
#pragma unroll
                    for (int i = 0; i < NH; ++i)
                        if (kb + i < lo || kb + i > hi) s_[i] = -INFINITY;
                }
                float m4[4] = {s_[0], s_[1], s_[2], s_[3]};
#pragma unroll
                for (int i = 4; i < NH; ++i) m4[i & 3] = fmaxf(m4[i & 3], s_[i]);
                sm.red_max[st][half][r] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                named_bar(bar_pair, 64);
                const float mx = fmaxf(sm.red_max[st][0][r], sm.red_max[st][1][r]);
                const float m_new = fmaxf(m_run, mx * c);
                const float m_use = m_new == -INFINITY ? 0.0f : m_new;
                const float corr = ex2_fast(m_run - m_use);
                float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < NH; ++i) {
                    s_[i] = ex2_fast(fmaf(s_[i], c, -m_use));
                    l4[i & 3] += s_[i];
                }
                l = fmaf(l, corr, (l4[0] + l4[1]) + (l4[2] + l4[3]));
                m_run = m_new;
                // P buffer st is free: o_full of tile n-2 was waited in its fold
                // P row r, keys 8*kc .. 8*kc+7 -> core matrix (r/8, kc): byte
                // (r/8)*(NK*16) + kc*128 + (r%8)*16
                uint8_t* prow = sm.p[st] + (r >> 3) * (NK * 16) + (r & 7) * 16 + half * (NH / 8) * 128;
#pragma unroll
                for (int kc = 0; kc < NH / 8; ++kc)
                    *reinterpret_cast<uint4*>(prow + kc * 128) = pack8(s_ + 8 * kc);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.p_full[st]);
                if (j > 0 && !fold(n - 1, corr_pending)) { ok = false; break; }
                corr_pending = corr;
            }
            if (!ok || !(ok = fold(n - 1, corr_pending))) break;  // the tile's last key tile
            // row sum over both halves (a slot per query-tile parity: the partner
            // may still read the previous tile's)
            sm.red_sum[qi & 1][half][r] = l;
            named_bar(bar_pair, 64);
            l = sm.red_sum[qi & 1][0][r] + sm.red_sum[qi & 1][1][r];
            if (t < T) {
                const float inv = l > 0.0f ? 1.0f / l : 0.0f;
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                                      ((size_t)tq.bh * T + t) * DV + half * DH);
#pragma unroll
                for (int j8 = 0; j8 < DH / 8; ++j8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = o[8 * j8 + e] * inv;
                    dst[j8] = pack8(y);
                }
            }
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

// Ring-cache fill after a forward over positions 0..T-1: the last min(T, w)
// keys and values go to slot (position mod w); pos[b] = T.  One thread per
// 16-byte piece of a row.
__global__ void ska_cache_fill_kernel(const SkaParams p) {
    const int n = min(p.T, p.window);
    const int kp = p.dk / 8, vp = p.dv / 8;  // 16-byte pieces per row
    const long long nk = p.k_cache ? (long long)p.B * n * kp : 0;
    const long long nv = p.v_cache ? (long long)p.B * p.H * n * vp : 0;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nk + nv;
         i += (long long)gridDim.x * blockDim.x) {
        if (i < nk) {
            const int x = (int)(i % kp);
            const long long row = i / kp;
            const int b = (int)(row / n), u = (int)(row % n);
            const int pos = p.T - n + u, slot = pos % p.window;
            const uint4* src = reinterpret_cast<const uint4*>(p.k) + ((size_t)b * p.T + pos) * kp + x;
            reinterpret_cast<uint4*>(p.k_cache)[((size_t)b * p.window + slot) * kp + x] = __ldg(src);
        } else {
            const long long j = i - nk;
            const int x = (int)(j % vp);
            const long long row = j / vp;
            const long long bh = row / n;
            const int u = (int)(row % n);
            const int pos = p.T - n + u, slot = pos % p.window;
            const uint4* src = reinterpret_cast<const uint4*>(p.v) + ((size_t)bh * p.T + pos) * vp + x;
            reinterpret_cast<uint4*>(p.v_cache)[((size_t)bh * p.window + slot) * vp + x] = __ldg(src);
        }
    }
    if (p.pos && blockIdx.x == 0)
        for (int b = threadIdx.x; b < p.B; b += blockDim.x) p.pos[b] = p.T;
}

// ------------------------------------------------------------------ decode
constexpr int kDecThreads = 256;

// dynamic shared memory of a decode CTA: G rows of scores, then the slot
// lanes' partial outputs
size_t ska_decode_smem_g(int window, int dv, int G) {
    return ((size_t)G * window + (size_t)(kDecThreads / (dv / 8)) * dv) * 4;
}

// G block-wide reductions at once (max or sum of v[g] over the CTA's threads);
// the results land in out[g] (shared memory) for every thread.  Two barriers:
// `red` is free again when the next call writes it.
template <int G>
__device__ __forceinline__ void block_reduce_g(float* v, float (*red)[kDecThreads / 32], float* out,
                                               bool is_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float x = v[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float y = __shfl_xor_sync(0xffffffffu, x, o);
            x = is_max ? fmaxf(x, y) : x + y;
        }
        if (lane == 0) red[g][warp] = x;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float x = red[threadIdx.x][0];
#pragma unroll
        for (int w = 1; w < kDecThreads / 32; ++w)
            x = is_max ? fmaxf(x, red[threadIdx.x][w]) : x + red[threadIdx.x][w];
        out[threadIdx.x] = x;
    }
    __syncthreads();
}

// One CTA per (b, group of G heads).  Valid slots are 0..n-1, n = min(pos+1, w)
// (before the ring fills, slot = position); the current token's slot takes
// the new key and value from the inputs, and this CTA writes them into the
// caches (the key by the group of head 0 only; no CTA reads that slot from the
// cache).  Each key row is read once for the G heads of the group.
template <int DK, int DV, int G>
__global__ void __launch_bounds__(kDecThreads) ska_decode_kernel(const SkaDecodeParams p) {
    extern __shared__ float dsm[];
    constexpr int XP = DV / 8, LG = kDecThreads / XP;   // value pieces, slot lanes
    float* sc = dsm;                       // [G][w] scores, then weights
    float* part = dsm + G * p.window;      // [LG][DV] partial outputs
    __shared__ __align__(16) float qs[G][DK];
    __shared__ float red[G][kDecThreads / 32];
    __shared__ float stat[2][G];           // row maximum, row sum
    const int ng = p.H / G;
    const int b = blockIdx.x / ng, h0 = (blockIdx.x % ng) * G;
    const int pos = p.pos[b];
    if (pos < 0) {  // the whole CTA leaves; nothing is read or written
        if (threadIdx.x == 0) atomicOr(p.err, kErrBadValue);
        return;
    }
    const int w = p.window, n = min(pos + 1, w), cur = pos % w;
    const size_t bh0 = (size_t)b * p.H + h0;
    const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(p.k) + (size_t)b * DK;
    const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(p.v) + bh0 * DV;
    const __nv_bfloat16* kc = static_cast<const __nv_bfloat16*>(p.k_cache) + (size_t)b * w * DK;
    const __nv_bfloat16* vc = static_cast<const __nv_bfloat16*>(p.v_cache) + bh0 * w * DV;
    const float c = p.scale * kLog2e;
    // start the shared key rows toward L2 once per sequence (the group of head
    // 0); prefetching the value rows as well measured slower (they evict one
    // another: the groups' value rows far exceed L2)
    if (threadIdx.x == 0 && h0 == 0) bulk_prefetch_l2(kc, (uint32_t)n * DK * 2);
    for (int i = threadIdx.x; i < G * DK; i += kDecThreads)
        qs[i / DK][i % DK] =
            __bfloat162float(static_cast<const __nv_bfloat16*>(p.q)[bh0 * DK + i]) * c;
    if (h0 == 0)
        for (int i = threadIdx.x; i < DK / 8; i += kDecThreads)
            reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.k_cache) + ((size_t)b * w + cur) * DK)[i] =
                reinterpret_cast<const uint4*>(kin)[i];
    for (int i = threadIdx.x; i < G * (DV / 8); i += kDecThreads) {
        const int g = i / (DV / 8), x = i % (DV / 8);
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.v_cache) + ((bh0 + g) * w + cur) * DV)[x] =
            reinterpret_cast<const uint4*>(vin + (size_t)g * DV)[x];
    }
    __syncthreads();
    // scores (log2 units): one slot per thread, its key row read once for G heads
    float mx[G];
#pragma unroll
    for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
    for (int u = threadIdx.x; u < n; u += kDecThreads) {
        const uint4* kr = reinterpret_cast<const uint4*>(u == cur ? kin : kc + (size_t)u * DK);
        float a[G];
#pragma unroll
        for (int g = 0; g < G; ++g) a[g] = 0.0f;
#pragma unroll 4
        for (int x = 0; x < DK / 8; ++x) {
            float f[8];
            unpack8(__ldg(kr + x), f);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                // the group's queries as two 16-byte shared-memory broadcasts
                const float4 qa = *reinterpret_cast<const float4*>(&qs[g][8 * x]);
                const float4 qb = *reinterpret_cast<const float4*>(&qs[g][8 * x + 4]);
                a[g] = fmaf(qa.x, f[0], a[g]); a[g] = fmaf(qa.y, f[1], a[g]);
                a[g] = fmaf(qa.z, f[2], a[g]); a[g] = fmaf(qa.w, f[3], a[g]);
                a[g] = fmaf(qb.x, f[4], a[g]); a[g] = fmaf(qb.y, f[5], a[g]);
                a[g] = fmaf(qb.z, f[6], a[g]); a[g] = fmaf(qb.w, f[7], a[g]);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            sc[g * w + u] = a[g];
            mx[g] = fmaxf(mx[g], a[g]);
        }
    }
    block_reduce_g<G>(mx, red, stat[0], true);
    float sum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sum[g] = 0.0f;
    for (int u = threadIdx.x; u < n; u += kDecThreads)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float e = ex2_fast(sc[g * w + u] - stat[0][g]);
            sc[g * w + u] = e;
            sum[g] += e;
        }
    block_reduce_g<G>(sum, red, stat[1], false);  // its barriers also publish sc
    // weighted sum of value rows, head by head: thread = (slot lane lg, 8-column piece x)
    const int x = threadIdx.x % XP, lg = threadIdx.x / XP;
    for (int g = 0; g < G; ++g) {
        const uint4* vbase = reinterpret_cast<const uint4*>(vc + (size_t)g * w * DV);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        // eight rows in flight per thread; plain (coherent) loads, since this CTA
        // wrote the new token's row into slot cur before the barrier above
        int u = lg;
        for (; u + 7 * LG < n; u += 8 * LG) {
            uint4 wv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) wv[j] = vbase[(size_t)(u + j * LG) * XP + x];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float f[8];
                unpack8(wv[j], f);
                const float pu = sc[g * w + u + j * LG];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(pu, f[e], acc[e]);
            }
        }
        for (; u < n; u += LG) {
            float f[8];
            unpack8(vbase[(size_t)u * XP + x], f);
            const float pu = sc[g * w + u];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(pu, f[e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) part[lg * DV + 8 * x + e] = acc[e];
        __syncthreads();
        const float inv = 1.0f / stat[1][g];
        for (int j = threadIdx.x; j < DV; j += kDecThreads) {
            float a = 0.0f;
            for (int l2 = 0; l2 < LG; ++l2) a += part[l2 * DV + j];
            static_cast<__nv_bfloat16*>(p.o)[(bh0 + g) * DV + j] = __float2bfloat16_rn(a * inv);
        }
        __syncthreads();  // part is rewritten by the next head
    }
}

__global__ void ska_advance_kernel(int* pos, int B) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) pos[b] += 1;
}

template <int DK, int DV>
cudaError_t launch_fwd_cfg(const SkaParams& p, cudaStream_t s) {
    using Kc = SkaCfg<DK, DV>;
    SkaKernelArgs a;
    a.p = p;
    const uint64_t BH = (uint64_t)p.B * p.H;
    if (!make_tmap_bf16_3d(&a.mq, p.q, DK, p.T, BH, 64, kQRows) ||
        !make_tmap_bf16_3d(&a.mk, p.k, DK, p.T, p.B, 64, Kc::NK) ||
        !make_tmap_bf16_3d(&a.mv, p.v, DV, p.T, BH, 64, Kc::NK))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(SkaSmem<DK, DV>) + 1024;
    auto kern = ska_fwd_kernel<DK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // One CTA per SM (d_k or d_v = 128): persistent CTAs, each walking about
    // tiles / SMs query tiles (measured 10-15% faster than a CTA per tile).
    // Two CTAs per SM: one query tile per CTA, so the many short CTAs balance
    // across SMs (persistent CTAs there measured 2% slower at window 512 and
    // 14% at window 2048: 5 or 6 tiles per CTA leave SMs idle at the end).
    const long long tiles = (long long)BH * ((p.T + kQRows - 1) / kQRows);
    const long long cap = Kc::CTAS_PER_SM == 1 ? (long long)sm_count() : tiles;
    kern<<<(unsigned)(tiles < cap ? tiles : cap), kSkaThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV, int G>
cudaError_t launch_dec_g(const SkaDecodeParams& p, cudaStream_t s) {
    const size_t smem = ska_decode_smem_g(p.window, DV, G);
    auto kern = ska_decode_kernel<DK, DV, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.B * (p.H / G)), kDecThreads, smem, s>>>(p);
    return cudaGetLastError();
}

// Heads per CTA: 8 where they divide H and their scores fit shared memory
// (each key row is then read once for eight heads; measured on B256 H16
// d 128 window 512: 216 us per step with one head per CTA, 167 with four, 122
// with eight, 150 with all sixteen, where 256 CTAs leave SMs idle), else 4, 2, 1.
template <int DK, int DV>
cudaError_t launch_dec_cfg(const SkaDecodeParams& p, cudaStream_t s) {
    constexpr size_t kFit = 200u << 10;
    if (p.H % 8 == 0 && ska_decode_smem_g(p.window, DV, 8) <= kFit) return launch_dec_g<DK, DV, 8>(p, s);
    if (p.H % 4 == 0 && ska_decode_smem_g(p.window, DV, 4) <= kFit) return launch_dec_g<DK, DV, 4>(p, s);
    if (p.H % 2 == 0 && ska_decode_smem_g(p.window, DV, 2) <= kFit) return launch_dec_g<DK, DV, 2>(p, s);
    return launch_dec_g<DK, DV, 1>(p, s);
}

}  // namespace


cudaError_t launch_ska_fwd(const SkaParams& p, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (p.T > 0) {
        if (p.dk == 64)
            e = p.dv == 64 ? launch_fwd_cfg<64, 64>(p, s) : launch_fwd_cfg<64, 128>(p, s);
        else
            e = p.dv == 64 ? launch_fwd_cfg<128, 64>(p, s) : launch_fwd_cfg<128, 128>(p, s);
        if (e != cudaSuccess) return e;
    }
    if (p.k_cache || p.v_cache || p.pos) {
        const long long n = p.T < p.window ? p.T : p.window;
        const long long work = (long long)p.B * n * (p.dk / 8 + (long long)p.H * (p.dv / 8));
        const long long blocks = (work + 255) / 256;
        const unsigned grid = (unsigned)(blocks < 1 ? 1 : blocks > 4 * 148 * 8 ? 4 * 148 * 8 : blocks);
        ska_cache_fill_kernel<<<grid, 256, 0, s>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

cudaError_t launch_ska_decode(const SkaDecodeParams& p, cudaStream_t s) {
    cudaError_t e;
    if (p.dk == 64)
        e = p.dv == 64 ? launch_dec_cfg<64, 64>(p, s) : launch_dec_cfg<64, 128>(p, s);
    else
        e = p.dv == 64 ? launch_dec_cfg<128, 64>(p, s) : launch_dec_cfg<128, 128>(p, s);
    if (e != cudaSuccess || !p.advance) return e;
    ska_advance_kernel<<<(p.B + 255) / 256, 256, 0, s>>>(p.pos, p.B);
    return cudaGetLastError();
}

}  // namespace rdm
