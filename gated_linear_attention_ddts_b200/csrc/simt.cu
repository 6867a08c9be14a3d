// simt.cu -- exact token-serial DDTS recurrence on CUDA cores (float32
// arithmetic, float32 or bf16 storage).  This is the float32 path and the
// path for shapes the tensor-core kernels do not take.
//
// Forward (per (b,h), one block; thread j owns column j of the state):
//     S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t k_t)(beta_hat_t v_t)^T,  o_t = S_t^T q_t
// (Rodimus*, digest.lyk-ai.com summary "Method" for the gates; diagonal decay
// along d_k per the paperhub.cn rebuttal "Efficient Parallelization" bullet.)
//
// Backward, exact reverse mode organised in two sweeps per (b,h), each run by a
// cluster of blocks that split the state's columns, TPR consecutive threads (8,
// or 4 at d_k = 128) owning row i of their block's columns of the state or of
// its gradient:
//   sweep F (forward in t):  S_t, dq_t = S_t dO_t (kept in float32 scratch too);
//   sweep R (reverse in t):  dS_t = q_t dO_t^T + diag(alpha_{t+1}) dS_{t+1},
//                            dkhat_t = dS_t vhat_t, dvhat_t = dS_t^T khat_t.
// The decay gradient uses d(log alpha_t) = sum_{u>=t} dG_u with
//   dG_u = q_u*dq_u - khat_u*dkhat_u  (+ rowsum(dS_T o S_T) at u = T),
// which follows from S_t = sum_s diag(exp(G_t - G_s)) khat_s vhat_s^T + diag(exp(G_t)) S_0
// with G_t the running sum of log alpha.
#include <cooperative_groups.h>
#include <type_traits>

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
// The state's columns are split over a cluster of DV / kCB blocks: the
// recurrences of dS and S act column by column, so each block runs its kCB
// columns for every row on its own.  Only the row sums over all columns (dq_t
// here, dkhat_t in sweep R) need the whole cluster; each block writes its
// partial sums of a tile of tokens into its shared memory, and after one cluster
// barrier per tile the block that owns a row adds the partials of every block
// through distributed shared memory, one (row, token) a thread.  The inputs of a
// tile are fetched one tile ahead with asynchronous copies, so their latency
// overlaps the tile before, and the tile's gate arithmetic is done once per
// (token, row) by the whole block before its token loop.
constexpr int kCB = 16;      // state columns per block
// Threads a row, TPR (a template parameter: 8 for d_k <= 64, 4 for d_k = 128,
// so a block has at most 512 threads), each running CH = kCB / TPR columns.
constexpr int kMaxRows = 128;

template <int DV>
__device__ __forceinline__ int owner_rows(int dk) {
    constexpr int NCB = DV / kCB;
    return (dk + NCB - 1) / NCB;
}

__host__ __device__ __forceinline__ int ntiles_of(int T) { return (T + kTile - 1) / kTile; }

// Sequence segments of the sweeps.  A head's tokens are cut into P segments of
// seg_len tokens (a multiple of kTile; the last one may be shorter), run by P
// clusters side by side.  Both recurrences are affine across a segment:
//   sweep F:  S_out = diag(e^L) S_in + S_loc,
//   sweep R:  C_out = diag(e^L) C_in + C_loc,  C = alpha_{t+1} o dS_{t+1} at a cut,
// with L the sum of log alpha over the segment's tokens and S_loc, C_loc the
// results from a zero start.  So a pass computes S_loc / C_loc and L of every
// segment (mode kSegLocal), and the full pass (kSegFull) of a segment folds the
// maps before it (F) or after it (R) onto S_0 / dS_T and runs from there.  The
// decay-gradient carry into segment j from later segments, fin + the sum of
// their dG totals, is added afterwards to dg and dtau of segment j by a fix-up
// launch.  P = 1 is the plain sweep.
enum { kSegWhole = 0, kSegLocal = 1, kSegFull = 2 };
struct SimtSeg {
    int P, seg_len, mode;
    float* Sx;   // [B H][P][d_k][d_v]: S_loc (sweep F), then C_loc (sweep R)
    float* La;   // [B H][P][d_k]: sum of log alpha over the segment
    float* tot;  // [B H][P][d_k]: the segment's sum of dG (sweep R)
};

// the two halves of a cluster barrier: arrive (releasing this thread's earlier
// writes, shared memory included) and wait (acquiring those of every thread
// that arrived); every thread of every block takes both
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// 16-byte global -> shared copies that complete asynchronously (cp.async), in
// per-thread commit groups
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// waits until at most the newest of this thread's groups is still in flight
__device__ __forceinline__ void cp_async_wait_prev() {
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

// One stage of the tile pipeline in dynamic shared memory, inputs as stored:
// the rows [kTile][dk] of g, tau, k, q, in sweep R the rows of dq (float32),
// then the block's columns [kTile][kCB] of beta, v, dO.  Every part is a
// multiple of 16 bytes (dk >= 16).
template <typename T>
struct SweepStage {
    T* row[4];
    float* dqf;
    T* col[3];
};

template <typename T>
__host__ __device__ __forceinline__ size_t sweep_stage_bytes(int dk, bool with_dq) {
    return (size_t)4 * kTile * dk * sizeof(T) + (with_dq ? (size_t)kTile * dk * 4 : 0) +
           (size_t)3 * kTile * kCB * sizeof(T);
}

template <typename T>
__device__ __forceinline__ SweepStage<T> sweep_stage(unsigned char* base, int dk, bool with_dq) {
    SweepStage<T> s;
    const size_t rb = (size_t)kTile * dk * sizeof(T), cb = (size_t)kTile * kCB * sizeof(T);
#pragma unroll
    for (int a = 0; a < 4; ++a) s.row[a] = reinterpret_cast<T*>(base + a * rb);
    unsigned char* p = base + 4 * rb;
    s.dqf = with_dq ? reinterpret_cast<float*>(p) : nullptr;
    if (with_dq) p += (size_t)kTile * dk * 4;
#pragma unroll
    for (int a = 0; a < 3; ++a) s.col[a] = reinterpret_cast<T*>(p + a * cb);
    return s;
}

// Starts the copies of tokens [t0, t0 + nt) into stage `st` (the rows of a tile
// are contiguous in [T][dk]; the block's kCB columns of a token are kCB * size
// bytes of [T][DV]) and closes one commit group; the rest of a partial tile is
// zero-filled with plain stores.  All addresses are 16-byte aligned: the
// pointers are, and every offset is a multiple of 16 * dk, DV or kCB elements.
template <typename T, int DV>
__device__ __forceinline__ void sweep_fetch(const SweepStage<T>& st, const T* const (&rows)[4],
                                            const float* dqf_bh, const T* const (&cols)[3], int t0,
                                            int nt, int dk) {
    const size_t roff = (size_t)t0 * dk;
    const int rchunks = nt * dk * (int)sizeof(T) / 16;
    for (int c = threadIdx.x; c < rchunks; c += blockDim.x) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
            cp_async16(reinterpret_cast<char*>(st.row[a]) + c * 16,
                       reinterpret_cast<const char*>(rows[a] + roff) + c * 16);
    }
    if (st.dqf) {
        for (int c = threadIdx.x; c < nt * dk / 4; c += blockDim.x)
            cp_async16(st.dqf + c * 4, dqf_bh + roff + c * 4);
    }
    constexpr int cpt = kCB * (int)sizeof(T) / 16;  // 16-byte pieces of one token's columns
    for (int c = threadIdx.x; c < nt * cpt; c += blockDim.x) {
        const int tt = c / cpt, part = c % cpt;
        const size_t off = (size_t)(t0 + tt) * DV;
#pragma unroll
        for (int a = 0; a < 3; ++a)
            cp_async16(reinterpret_cast<char*>(st.col[a] + tt * kCB) + part * 16,
                       reinterpret_cast<const char*>(cols[a] + off) + part * 16);
    }
    cp_async_commit();
    if (nt < kTile) {
        for (int e = nt * dk + threadIdx.x; e < kTile * dk; e += blockDim.x) {
#pragma unroll
            for (int a = 0; a < 4; ++a) stf(st.row[a] + e, 0.0f);
            if (st.dqf) st.dqf[e] = 0.0f;
        }
        for (int e = nt * kCB + threadIdx.x; e < kTile * kCB; e += blockDim.x) {
#pragma unroll
            for (int a = 0; a < 3; ++a) stf(st.col[a] + e, 0.0f);
        }
    }
}

// Sweep F of head bh, segment sj, by this cluster.
template <typename T, int DV, int TPR>
__device__ __forceinline__ void fsweep_head(const BwdParams& p, float* dqf, float* fin,
                                            const SimtSeg& sg, int bh, int sj) {
    constexpr int NCB = DV / kCB, CH = kCB / TPR;
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank(), cid = bh * sg.P + sj;
    if (sg.mode == kSegLocal && sj == sg.P - 1) return;  // the last segment's map is never used
    const bool local = sg.mode == kSegLocal;
    const int T_ = p.T, dk = p.dk, c0 = rank * kCB;
    const int sa = sj * sg.seg_len, sb = min(T_, sa + sg.seg_len);  // this segment's tokens
    // TPR threads a row: thread TPR i + h runs columns c0 + CH h ... c0 + CH (h + 1) - 1
    // of row i (the block has TPR d_k threads)
    const int i = threadIdx.x / TPR, cb = (threadIdx.x % TPR) * CH;
    const bool act = i < dk;
    const int rows_pb = owner_rows<DV>(dk), r0 = rank * rows_pb;  // rows this block finishes
    __shared__ float s_vh[kTile][kCB], s_do[kTile][kCB], s_part[2][kTile][kMaxRows], s_fin[kMaxRows];
    extern __shared__ __align__(16) unsigned char s_stage[];

    const size_t rbase = (size_t)bh * T_ * dk, cbase = (size_t)bh * T_ * DV + c0;
    const T* const rows[4] = {static_cast<const T*>(p.g) + rbase, static_cast<const T*>(p.tau) + rbase,
                              static_cast<const T*>(p.k) + rbase, static_cast<const T*>(p.q) + rbase};
    const T* const cols[3] = {static_cast<const T*>(p.beta) + cbase, static_cast<const T*>(p.v) + cbase,
                              static_cast<const T*>(p.dO) + cbase};
    T* dq = static_cast<T*>(p.dq) + rbase;
    float* dqf_bh = dqf + rbase;
    const size_t sbytes = sweep_stage_bytes<T>(dk, false);
    // the tile's gates as the token loop uses them, [kTile][dk]: alpha and
    // khat = alpha_hat k (1 and 0 past the end of a partial tile)
    float* s_al = reinterpret_cast<float*>(s_stage + 2 * sbytes);
    float* s_kh = s_al + kTile * dk;
    float* s_la = s_kh + kTile * dk;  // log alpha (0 past the end), for a local pass
    float* Sx = sg.Sx + ((size_t)cid * dk + i) * DV + c0 + cb;  // this thread's part of the segment's slot

    // the segment's entry state: zero for a local pass, else S_0 folded through
    // the maps of the segments before this one (S_in(j+1) = diag(e^{L_j}) S_in(j)
    // + S_loc(j); none for the whole sequence or the first segment)
    float s[CH], lsum = 0.0f;
#pragma unroll
    for (int j = 0; j < CH; ++j)
        s[j] = !act || local || !p.S0 ? 0.0f : p.S0[((size_t)bh * dk + i) * DV + c0 + cb + j];
    if (act && !local) {
        for (int jj = 0; jj < sj; ++jj) {
            const size_t slot = (size_t)bh * sg.P + jj;
            const float e = expf(sg.La[slot * dk + i]);
            const float* loc = sg.Sx + (slot * dk + i) * DV + c0 + cb;
#pragma unroll
            for (int j = 0; j < CH; ++j) s[j] = fmaf(e, s[j], loc[j]);
        }
    }

    // Tile n: its stage was fetched while tile n - 1 ran; it is unpacked into
    // s_vh, s_do and the gate arrays before the cluster waits for the partial
    // sums of tile n - 1, so that wait overlaps the unpacking.
    auto fetch = [&](int m) {  // starts tile m's copies (an empty group past the end)
        if (m < ntiles_of(sb - sa)) {
            const int tm = sa + m * kTile;
            sweep_fetch<T, DV>(sweep_stage<T>(s_stage + (m & 1) * sbytes, dk, false), rows, nullptr,
                               cols, tm, min(kTile, sb - tm), dk);
        } else {
            cp_async_commit();
        }
    };
    auto unpack = [&](int m) {  // after tile m's copies are complete and visible
        const SweepStage<T> cur = sweep_stage<T>(s_stage + (m & 1) * sbytes, dk, false);
        const int nt_m = min(kTile, sb - sa - m * kTile);
        for (int idx = threadIdx.x; idx < kTile * kCB; idx += blockDim.x) {
            const float bb = ldf(cur.col[0] + idx);
            s_vh[idx / kCB][idx % kCB] = (p.preact ? sigmoid_acc(bb) : bb) * ldf(cur.col[1] + idx);
            s_do[idx / kCB][idx % kCB] = ldf(cur.col[2] + idx);
        }
        // the gate arithmetic of every (token, row) once, spread over the block
        for (int e = threadIdx.x; e < kTile * dk; e += blockDim.x) {
            float gg = ldf(cur.row[0] + e), ta = ldf(cur.row[1] + e);
            if (p.preact) {
                gg = softplus_acc(gg);
                ta = sigmoid_acc(ta);
            }
            const bool live = e / dk < nt_m;
            s_al[e] = live ? alpha(gg, ta) : 1.0f;
            s_kh[e] = live ? alpha_hat(gg, ta) * ldf(cur.row[2] + e) : 0.0f;
            s_la[e] = live ? log_alpha(gg, ta) : 0.0f;
        }
    };
    const int ntiles = ntiles_of(sb - sa);
    if (ntiles > 0) {
        fetch(0);
        fetch(1);
        cp_async_wait_prev();
        __syncthreads();
        unpack(0);
        __syncthreads();
    }
    for (int n = 0; n < ntiles; ++n) {
        const int t0 = sa + n * kTile, nt = min(kTile, sb - t0), buf = n & 1;
        if (local) {
            // the segment's map only: the state from zero and the sum of log alpha
#pragma unroll
            for (int tt = 0; tt < kTile; ++tt) {
                const float al = s_al[tt * dk + i], kh = s_kh[tt * dk + i];
                lsum += s_la[tt * dk + i];
#pragma unroll
                for (int j = 0; j < CH; ++j) s[j] = fmaf(al, s[j], kh * s_vh[tt][cb + j]);
            }
            if (n + 1 < ntiles) {
                fetch(n + 2);
                cp_async_wait_prev();
                __syncthreads();
                unpack(n + 1);
                __syncthreads();
            }
            continue;
        }
        // the tile's tokens as one straight run (a token past the end of a partial
        // tile leaves the state as it is: alpha 1, khat 0)
#pragma unroll
        for (int tt = 0; tt < kTile; ++tt) {
            const float al = s_al[tt * dk + i], kh = s_kh[tt * dk + i];
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int j = 0; j < CH; j += 2) {
                s[j] = fmaf(al, s[j], kh * s_vh[tt][cb + j]);
                s[j + 1] = fmaf(al, s[j + 1], kh * s_vh[tt][cb + j + 1]);
                a0 = fmaf(s[j], s_do[tt][cb + j], a0);
                a1 = fmaf(s[j + 1], s_do[tt][cb + j + 1], a1);
            }
            float a = a0 + a1;
#pragma unroll
            // the row's other columns
            for (int o = 1; o < TPR; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (act && cb == 0) s_part[buf][tt][i] = a;
        }
        // this block's partials of the tile are written (s_part alternates by tile:
        // a block writes tile n + 2 into this buffer only after every block has
        // arrived after tile n + 1, that is, after it read tile n's sums)
        cluster_arrive();
        if (n + 1 < ntiles) {
            fetch(n + 2);  // into the stage tile n came from, unpacked before its run
            cp_async_wait_prev();
            __syncthreads();  // tile n + 1's stage is visible; tile n's run is over
            unpack(n + 1);
            __syncthreads();
        }
        cluster_wait();  // every block's partials of tile n are written
        // dq of this block's rows, one (row, token) a thread: the sum of every
        // block's partial through distributed shared memory
        for (int it = threadIdx.x; it < rows_pb * kTile; it += blockDim.x) {
            const int row = r0 + it / kTile, tt = it % kTile;
            if (row < dk && tt < nt) {
                float acc = 0.0f;
#pragma unroll
                for (int r = 0; r < NCB; ++r) acc += *cl.map_shared_rank(&s_part[buf][tt][row], r);
                const size_t off = (size_t)(t0 + tt) * dk + row;
                stf(dq + off, acc);
                dqf_bh[off] = acc;
            }
        }
    }
    if (local) {  // the segment's map: S_loc (this thread's columns) and L (its row)
        if (act) {
#pragma unroll
            for (int j = 0; j < CH; ++j) Sx[j] = s[j];
            if (cb == 0) sg.La[(size_t)cid * dk + i] = lsum;
        }
        return;
    }
    if (sj != sg.P - 1) {
        cl.sync();  // no block leaves while another still reads its shared memory
        return;
    }
    // rowsum(dS_T o S_T), the decay gradient's term at u = T
    float f = 0.0f;
    if (act && p.dST) {
#pragma unroll
        for (int j = 0; j < CH; ++j)
            f = fmaf(p.dST[((size_t)bh * dk + i) * DV + c0 + cb + j], s[j], f);
    }
#pragma unroll
    for (int o = 1; o < TPR; o <<= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
    if (act && cb == 0) s_fin[i] = f;
    cl.sync();
    for (int row = r0 + threadIdx.x; row < min(dk, r0 + rows_pb); row += blockDim.x) {
        float acc = 0.0f;
#pragma unroll
        for (int r = 0; r < NCB; ++r) acc += *cl.map_shared_rank(&s_fin[row], r);
        fin[(size_t)bh * dk + row] = acc;
    }
    cl.sync();  // no block leaves while another still reads its shared memory
}

// ------------------------------------------------ backward, reverse sweep R
// Sweep R of head bh, segment sj, by this cluster.
template <typename T, int DV, int TPR>
__device__ __forceinline__ void rsweep_head(const BwdParams& p, const float* dqf, const float* fin,
                                            const SimtSeg& sg, int bh, int sj) {
    constexpr int NCB = DV / kCB, CH = kCB / TPR;
    static_assert(TPR == 4 || TPR == 8, "the column reduce-scatter below takes CH = 4 or 2");
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank(), cid = bh * sg.P + sj;
    if (sg.mode == kSegLocal && sj == 0) return;  // the first segment's map is never used
    const bool local = sg.mode == kSegLocal;
    const int T_ = p.T, dk = p.dk, c0 = rank * kCB;
    const int sa = sj * sg.seg_len, sb = min(T_, sa + sg.seg_len);  // this segment's tokens
    // TPR threads a row, as in sweep F
    const int i = threadIdx.x / TPR, cb = (threadIdx.x % TPR) * CH;
    const bool act = i < dk;
    const int rows_pb = owner_rows<DV>(dk), r0 = rank * rows_pb;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x / 32;
    __shared__ float s_vh[kTile][kCB], s_do[kTile][kCB], s_b[kTile][kCB], s_v[kTile][kCB];
    __shared__ float s_part[2][kTile][kMaxRows], s_red[kTile][16][kCB];
    __shared__ float s_da[kMaxRows];  // decay-gradient carry of this block's rows
    extern __shared__ __align__(16) unsigned char s_stage[];

    const size_t rbase = (size_t)bh * T_ * dk, cbase = (size_t)bh * T_ * DV + c0;
    const T* const rows[4] = {static_cast<const T*>(p.g) + rbase, static_cast<const T*>(p.tau) + rbase,
                              static_cast<const T*>(p.k) + rbase, static_cast<const T*>(p.q) + rbase};
    const T* const cols[3] = {static_cast<const T*>(p.beta) + cbase, static_cast<const T*>(p.v) + cbase,
                              static_cast<const T*>(p.dO) + cbase};
    T* dk_ = static_cast<T*>(p.dk_) + rbase;
    T* dg = static_cast<T*>(p.dg) + rbase;
    T* dtau = static_cast<T*>(p.dtau) + rbase;
    T* dv_ = static_cast<T*>(p.dv_) + cbase;
    T* dbeta = static_cast<T*>(p.dbeta) + cbase;
    const float* dqf_bh = dqf + rbase;
    const float* dfeed = p.dfeed ? p.dfeed + (size_t)(bh % p.H) * DV + c0 : nullptr;
    const size_t sbytes = sweep_stage_bytes<T>(dk, true);
    // the tile's gates, [kTile][dk] each: alpha and khat = alpha_hat k for the
    // token loop (1 and 0 past the end of a partial tile), and for the scan the
    // activated g and tau, alpha_hat and log2 g
    float* s_al = reinterpret_cast<float*>(s_stage + 2 * sbytes);
    float* s_kh = s_al + kTile * dk;
    float* s_gg = s_kh + kTile * dk;
    float* s_ta = s_gg + kTile * dk;
    float* s_ah = s_ta + kTile * dk;
    float* s_lg = s_ah + kTile * dk;

    float* Sx = sg.Sx + ((size_t)cid * dk + i) * DV + c0 + cb;  // this thread's part of the segment's slot

    // the gradient flowing in at the segment's end: zero for a local pass, else
    // dS_T (alpha_{T+1} taken as 1) folded through the maps of the segments after
    // this one (C_in(j-1) = diag(e^{L_j}) C_in(j) + C_loc(j))
    float ds[CH], lsum = 0.0f;
#pragma unroll
    for (int j = 0; j < CH; ++j)
        ds[j] = !act || local || !p.dST ? 0.0f : p.dST[((size_t)bh * dk + i) * DV + c0 + cb + j];
    if (act && !local) {
        for (int jj = sg.P - 1; jj > sj; --jj) {
            const size_t slot = (size_t)bh * sg.P + jj;
            const float e = expf(sg.La[slot * dk + i]);
            const float* loc = sg.Sx + (slot * dk + i) * DV + c0 + cb;
#pragma unroll
            for (int j = 0; j < CH; ++j) ds[j] = fmaf(e, ds[j], loc[j]);
        }
    }
    float a_next = 1.0f;  // alpha_{t+1,i}
    // the carry fin + later segments' dG enters the last segment here; the other
    // segments' carries are added by the fix-up launch
    const bool last = sj == sg.P - 1;
    for (int rl = threadIdx.x; rl < rows_pb; rl += blockDim.x)
        s_da[rl] = r0 + rl < dk && last ? fin[(size_t)bh * dk + r0 + rl] : 0.0f;

    // tile n holds tokens [t1 - kTile, t1) with t1 = sb - n kTile (the last one
    // processed may be partial)
    const int ntiles = ntiles_of(sb - sa);
    if (ntiles > 0)
        sweep_fetch<T, DV>(sweep_stage<T>(s_stage, dk, true), rows, dqf_bh, cols, max(sa, sb - kTile),
                           min(kTile, sb - sa), dk);
    for (int n = 0; n < ntiles; ++n) {
        const int t1 = sb - n * kTile, t0 = max(sa, t1 - kTile), nt = t1 - t0, buf = n & 1;
        const SweepStage<T> cur = sweep_stage<T>(s_stage + buf * sbytes, dk, true);
        if (n + 1 < ntiles)
            sweep_fetch<T, DV>(sweep_stage<T>(s_stage + (buf ^ 1) * sbytes, dk, true), rows, dqf_bh,
                               cols, max(sa, t0 - kTile), min(kTile, t0 - sa), dk);
        else
            cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();  // this tile's stage is complete and visible
        for (int idx = threadIdx.x; idx < kTile * kCB; idx += blockDim.x) {
            const int tt = idx / kCB, j = idx % kCB;
            const float b_in = ldf(cur.col[0] + idx), vv = ldf(cur.col[1] + idx);
            const float bb = p.preact ? sigmoid_acc(b_in) : b_in;
            s_b[tt][j] = bb;
            s_v[tt][j] = vv;
            s_vh[tt][j] = bb * vv;
            s_do[tt][j] = ldf(cur.col[2] + idx);
        }
        // the gate arithmetic of every (token, row) once, spread over the block
        for (int e = threadIdx.x; e < kTile * dk; e += blockDim.x) {
            float gg = ldf(cur.row[0] + e), ta = ldf(cur.row[1] + e);
            if (p.preact) {
                gg = softplus_acc(gg);
                ta = sigmoid_acc(ta);
            }
            const bool live = e / dk < nt;
            // alpha_hat = g^tau with 0^0 = 1 and 0^tau = 0 (log2(0) = -inf)
            const float lg = log2f(gg);
            const float ah = ta == 0.0f ? 1.0f : exp2f(ta * lg);
            s_al[e] = live ? alpha(gg, ta) : 1.0f;
            s_kh[e] = live ? ah * ldf(cur.row[2] + e) : 0.0f;
            s_gg[e] = gg;
            s_ta[e] = ta;
            s_ah[e] = ah;
            s_lg[e] = lg;
        }
        __syncthreads();
        if (local) {
            // the segment's map only: dS from zero and the sum of log alpha
#pragma unroll
            for (int tt = kTile - 1; tt >= 0; --tt) {
                const bool live = tt < nt;
                const float f = live ? a_next : 1.0f;
                const float qi = act ? ldf(cur.row[3] + tt * dk + i) : 0.0f;
#pragma unroll
                for (int j = 0; j < CH; ++j) ds[j] = fmaf(f, ds[j], qi * s_do[tt][cb + j]);
                if (live) {
                    lsum += log_alpha(s_gg[tt * dk + i], s_ta[tt * dk + i]);
                    a_next = s_al[tt * dk + i];
                }
            }
            __syncthreads();  // the staging buffers and gate arrays are free for the next tile
            continue;
        }
        // the tile's tokens as one straight run, as in sweep F (a token past the end
        // of a partial tile leaves dS as it is: factor 1, no q dO^T term)
#pragma unroll
        for (int tt = kTile - 1; tt >= 0; --tt) {
            const bool live = tt < nt;
            const float f = live ? a_next : 1.0f;
            const float qi = act ? ldf(cur.row[3] + tt * dk + i) : 0.0f;
            const float kh = act ? s_kh[tt * dk + i] : 0.0f;
            float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
            for (int j = 0; j < CH; j += 2) {
                ds[j] = fmaf(f, ds[j], qi * s_do[tt][cb + j]);
                ds[j + 1] = fmaf(f, ds[j + 1], qi * s_do[tt][cb + j + 1]);
                d0 = fmaf(ds[j], s_vh[tt][cb + j], d0);
                d1 = fmaf(ds[j + 1], s_vh[tt][cb + j + 1], d1);
            }
            float d = d0 + d1;
#pragma unroll
            // the row's other columns
            for (int o = 1; o < TPR; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (act && cb == 0) s_part[buf][tt][i] = d;  // this block's share of dkhat_{t,i}
            // dvhat_j = sum_i dS_ij khat_i over the warp's 32 / TPR rows (lanes with
            // the same l mod TPR): a reduce-scatter over the top lane bits (each
            // halving round sends half of the lane's partial sums to the lane `o`
            // apart and adds the other half it receives: bits 4, 3 for CH = 4, bit 4
            // for CH = 2), then a plain sum over the next bit (TPR), after which
            // lanes l and l ^ TPR both hold column cb + col; the warps meet below
            float x[CH / 2];
            const bool up0 = (lane & 16) != 0;
            int col = up0 ? CH / 2 : 0;
#pragma unroll
            for (int j = 0; j < CH / 2; ++j) {
                const float lo = ds[j] * kh, hi = ds[j + CH / 2] * kh;
                x[j] = (up0 ? hi : lo) + __shfl_xor_sync(0xffffffffu, up0 ? lo : hi, 16);
            }
            if constexpr (CH == 4) {
                const bool up = (lane & 8) != 0;
                x[0] = (up ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, up ? x[0] : x[1], 8);
                if (up) col += 1;
            }
            x[0] += __shfl_xor_sync(0xffffffffu, x[0], TPR);
            if ((lane & TPR) == 0) s_red[tt][warp][cb + col] = x[0];
            if (live) a_next = s_al[tt * dk + i];
        }
        // this block's dkhat partials of the tile are written (s_part alternates by
        // tile, as in sweep F); the dvhat outputs need only this block's partials
        cluster_arrive();
        __syncthreads();
        for (int idx = threadIdx.x; idx < nt * kCB; idx += blockDim.x) {
            const int tt = idx / kCB, j = idx % kCB;
            float dvh = 0.0f;
            for (int w = 0; w < nwarps; ++w) dvh += s_red[tt][w][j];
            const size_t ov = (size_t)(t0 + tt) * DV + j;
            const float bb = s_b[tt][j];
            const float df = dfeed ? dfeed[j] * s_do[tt][j] : 0.0f;
            stf(dv_ + ov, fmaf(bb, dvh, df));
            stf(dbeta + ov, (p.preact ? bb * (1.0f - bb) : 1.0f) * s_v[tt][j] * dvh);
        }
        cluster_wait();  // every block's dkhat partials of the tile are written
        // The decay gradient of this block's rows, one (row, token) a thread: the
        // 16 tokens of a row are 16 consecutive lanes (rows_pb * kTile = 16 d_k / NCB
        // items, a multiple of 32, so whole warps take a pass and shuffle).  d log alpha_t is the row's
        // carry (every later tile) plus the suffix sum over the tile's tokens u >= t
        // of dG_u = q_u dq_u - khat_u dkhat_u.
        for (int it = threadIdx.x; it < rows_pb * kTile; it += blockDim.x) {
            const int rl = it / kTile, row = min(r0 + rl, dk - 1), tt = it % kTile;
            const bool live = tt < nt && r0 + rl < dk;
            const int e = tt * dk + row;
            float dkh = 0.0f;
#pragma unroll
            for (int r = 0; r < NCB; ++r) dkh += *cl.map_shared_rank(&s_part[buf][tt][row], r);
            const float kk = ldf(cur.row[2] + e), ah = s_ah[e];
            const float dG = live ? ldf(cur.row[3] + e) * cur.dqf[e] - ah * kk * dkh : 0.0f;
            const float carry = s_da[rl];
            float sfx = dG;
#pragma unroll
            for (int o = 1; o < kTile; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, sfx, o, kTile);
                if (tt + o < kTile) sfx += y;
            }
            const float da = carry + sfx;
            const float gg = s_gg[e], ta = s_ta[e], lg = s_lg[e];
            // chain factors to the pre-activations: softplus' = sigmoid, which is
            // 1 - e^-g of the activated g; sigmoid' = s (1 - s)
            const float cg_ = p.preact ? -expm1f(-gg) : 1.0f;
            const float ct = p.preact ? ta * (1.0f - ta) : 1.0f;
            const float dah = kk * dkh;
            // d alpha_hat / d g = tau g^(tau - 1), which is tau alpha_hat / g while
            // alpha_hat is a normal number (then g > 0); d alpha_hat / d tau =
            // alpha_hat ln g
            const float dah_dg = ta == 0.0f ? 0.0f
                                 : ah >= 1.17549435e-38f ? __fdividef(ta * ah, gg)
                                                          : ta * exp2f((ta - 1.0f) * lg);
            const float dah_dtau = ah == 0.0f ? 0.0f : ah * (lg * kLn2);
            if (live) {
                const size_t off = (size_t)(t0 + tt) * dk + row;
                stf(dk_ + off, ah * dkh);
                stf(dg + off, cg_ * (-ta * da + dah_dg * dah));
                stf(dtau + off, ct * (-gg * da + dah_dtau * dah));
            }
            __syncwarp();  // every lane of the row has read the carry
            if (tt == 0) s_da[rl] = carry + sfx;  // the whole tile's sum
        }
        __syncthreads();  // the staging buffers, gate arrays and s_red are free for the next tile
    }
    if (local) {  // the segment's map: C_loc = alpha_{first} o dS_{first} and L
        if (act) {
#pragma unroll
            for (int j = 0; j < CH; ++j) Sx[j] = a_next * ds[j];
            if (cb == 0) sg.La[(size_t)cid * dk + i] = lsum;
        }
        return;
    }
    if (act && p.dS0 && sj == 0) {
#pragma unroll
        for (int j = 0; j < CH; ++j) p.dS0[((size_t)bh * dk + i) * DV + c0 + cb + j] = a_next * ds[j];
    }
    if (sg.mode == kSegFull) {  // the segment's sum of dG, for the carries of earlier segments
        for (int rl = threadIdx.x; rl < rows_pb; rl += blockDim.x)
            if (r0 + rl < dk)
                sg.tot[(size_t)cid * dk + r0 + rl] =
                    s_da[rl] - (last ? fin[(size_t)bh * dk + r0 + rl] : 0.0f);
    }
    cl.sync();  // no block leaves while another still reads its shared memory
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

// Programmatic dependent launch: a launch of the chain below may start while
// the one before it is finishing (its blocks then wait in chain_enter until that
// grid has completed and its writes are visible); a block lets the next launch
// start once it is done (chain_leave), so the waiting blocks never hold an SM
// that a working block of this launch could use.
__device__ __forceinline__ void chain_enter() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void chain_leave() {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// The sweep kernels: cluster c takes segment c % P of the heads slot, slot +
// slots, ... (slot = c / P) of `list` (list[0] heads, then their indices; every
// head when list is null).  The tensor-core backward lists only the heads it
// flagged, so a few slots cover them and the launch stays small.
template <typename T, int DV, int TPR>
__global__ void __launch_bounds__(512) simt_bwd_fsweep(const BwdParams p, float* dqf, float* fin,
                                                       const int* list, int slots, const SimtSeg sg) {
    chain_enter();
    const int c = blockIdx.x / (DV / kCB), slot = c / sg.P, sj = c % sg.P;
    const int nheads = list ? list[0] : p.B * p.H;
    for (int q = slot; q < nheads; q += slots) {
        fsweep_head<T, DV, TPR>(p, dqf, fin, sg, list ? list[1 + q] : q, sj);
        __syncthreads();
    }
    chain_leave();
}

template <typename T, int DV, int TPR>
__global__ void __launch_bounds__(512) simt_bwd_rsweep(const BwdParams p, const float* dqf,
                                                       const float* fin, const int* list, int slots,
                                                       const SimtSeg sg) {
    chain_enter();
    const int c = blockIdx.x / (DV / kCB), slot = c / sg.P, sj = c % sg.P;
    const int nheads = list ? list[0] : p.B * p.H;
    for (int q = slot; q < nheads; q += slots) {
        rsweep_head<T, DV, TPR>(p, dqf, fin, sg, list ? list[1 + q] : q, sj);
        __syncthreads();
    }
    chain_leave();
}

// list[0] = the number of flagged heads, list[1..] their indices (one block).
__global__ void simt_flag_list(const int* flags, int BH, int* list) {
    __shared__ int n;
    if (threadIdx.x == 0) n = 0;
    __syncthreads();
    for (int bh = threadIdx.x; bh < BH; bh += blockDim.x)
        if (flags[bh] != 0) list[1 + atomicAdd(&n, 1)] = bh;
    __syncthreads();
    if (threadIdx.x == 0) list[0] = n;
}

// One sweep launch (F when `rev` is false, R when true) in the segment mode of `sg`.
template <typename T, int DV, int TPR>
cudaError_t bwd_tvr(const BwdParams& p, float* dqf, float* fin, const int* list, int slots,
                    const SimtSeg& sg, bool rev, cudaStream_t s) {
    // one cluster of DV / kCB blocks per (b,h) and segment
    constexpr int NCB = DV / kCB;
    // two pipeline stages of dynamic shared memory (sweep R's carry dq too), then
    // the tile's gate arrays (three in sweep F, six in sweep R)
    const size_t ga = (size_t)kTile * p.dk * 4;
    const size_t sm = rev ? 2 * sweep_stage_bytes<T>(p.dk, true) + 6 * ga
                          : 2 * sweep_stage_bytes<T>(p.dk, false) + 3 * ga;
    cudaError_t e = rev ? cudaFuncSetAttribute(simt_bwd_rsweep<T, DV, TPR>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)
                        : cudaFuncSetAttribute(simt_bwd_fsweep<T, DV, TPR>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(slots * sg.P * NCB));
    cfg.blockDim = dim3((unsigned)(TPR * p.dk));
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = NCB;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    if (rev)
        return cudaLaunchKernelEx(&cfg, simt_bwd_rsweep<T, DV, TPR>, p, static_cast<const float*>(dqf),
                                  static_cast<const float*>(fin), list, slots, sg);
    return cudaLaunchKernelEx(&cfg, simt_bwd_fsweep<T, DV, TPR>, p, dqf, fin, list, slots, sg);
}

template <typename T, int DV>
cudaError_t bwd_tv(const BwdParams& p, float* dqf, float* fin, const int* list, int slots,
                   const SimtSeg& sg, bool rev, cudaStream_t s) {
    return p.dk <= 64 ? bwd_tvr<T, DV, 8>(p, dqf, fin, list, slots, sg, rev, s)
                      : bwd_tvr<T, DV, 4>(p, dqf, fin, list, slots, sg, rev, s);
}

template <typename T>
cudaError_t bwd_t(const BwdParams& p, float* dqf, float* fin, const int* list, int slots,
                  const SimtSeg& sg, bool rev, cudaStream_t s) {
    switch (p.dv) {
        case 16: return bwd_tv<T, 16>(p, dqf, fin, list, slots, sg, rev, s);
        case 32: return bwd_tv<T, 32>(p, dqf, fin, list, slots, sg, rev, s);
        case 64: return bwd_tv<T, 64>(p, dqf, fin, list, slots, sg, rev, s);
        case 128: return bwd_tv<T, 128>(p, dqf, fin, list, slots, sg, rev, s);
        default: return cudaErrorInvalidValue;
    }
}

// The fix-up launch: blocks [slot * kFixBlocks, (slot + 1) * kFixBlocks) take the
// heads slot, slot + slots, ... of the list (as the sweeps do).
constexpr int kFixBlocks = 128;

__device__ __forceinline__ int listed_heads(const int* list, int BH) { return list ? list[0] : BH; }
__device__ __forceinline__ int listed_head(const int* list, int q) { return list ? list[1 + q] : q; }

// dg and dtau of every segment but the last, plus the decay-gradient carry into
// it: fin + the dG sums of all later segments (d log alpha grows by that carry
// at every token of the segment).  One thread per
// (t, i) of the head.
template <typename T>
__global__ void simt_carry_fix(const BwdParams p, const SimtSeg sg, const float* fin,
                               const int* list, int slots) {
    chain_enter();
    const int dk = p.dk;
    const int n = min(p.T, (sg.P - 1) * sg.seg_len) * dk;
    for (int q = blockIdx.x / kFixBlocks; q < listed_heads(list, p.B * p.H); q += slots) {
        const int bh = listed_head(list, q);
        for (int e = (blockIdx.x % kFixBlocks) * blockDim.x + threadIdx.x; e < n;
             e += kFixBlocks * blockDim.x) {
            const int i = e % dk, t = e / dk;
            float carry = fin[(size_t)bh * dk + i];
            for (int j = t / sg.seg_len + 1; j < sg.P; ++j)
                carry += sg.tot[((size_t)bh * sg.P + j) * dk + i];
            const size_t off = ((size_t)bh * p.T + t) * dk + i;
            const float g_in = ldf(static_cast<const T*>(p.g) + off);
            const float t_in = ldf(static_cast<const T*>(p.tau) + off);
            const float gg = p.preact ? softplus_acc(g_in) : g_in;
            const float ta = p.preact ? sigmoid_acc(t_in) : t_in;
            const float cg = p.preact ? sigmoid_acc(g_in) : 1.0f;
            const float ct = p.preact ? ta * (1.0f - ta) : 1.0f;
            T* dg = static_cast<T*>(p.dg) + off;
            T* dtau = static_cast<T*>(p.dtau) + off;
            stf(dg, ldf(dg) - cg * ta * carry);
            stf(dtau, ldf(dtau) - ct * gg * carry);
        }
    }
}

// Segments of the exact backward: P = min(8, T / 512) for T >= 1024 (segments of
// at least 512 tokens), seg_len a whole number of tiles; the count actually used
// is the number of non-empty segments.
void simt_segments(int T, int* P, int* seg_len) {
    const int want = T >= 1024 ? min(8, T / 512) : 1;
    const int tiles = ntiles_of(T);
    const int len = max(1, (tiles + want - 1) / want) * kTile;
    *P = max(1, (T + len - 1) / len);
    *seg_len = *P > 1 ? len : max(T, 1);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

cudaError_t launch_simt_fwd(const SeqParams& p, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    return p.bf16 ? fwd_t<__nv_bfloat16>(p, s) : fwd_t<float>(p, s);
}

// scratch, float32: dq for every (b,h,t,i), the final-state term per (b,h,i),
// the flagged-head list (int32) and, with segments, the segments' state slots
// [B H][P][d_k][d_v], their sums of log alpha and of dG [B H][P][d_k]
size_t simt_bwd_workspace(const BwdParams& p) {
    int P, len;
    simt_segments(p.T, &P, &len);
    const size_t rows = (size_t)p.B * p.H * p.dk;
    size_t w = align256(rows * (size_t)p.T * 4) + align256(rows * 4) +
               align256((size_t)(p.B * p.H + 1) * 4);  // the flagged-head list
    if (P > 1) w += align256(rows * P * (size_t)p.dv * 4) + 2 * align256(rows * P * 4);
    return w;
}

// heads a launch of the flagged re-run covers side by side (more flagged heads
// run in turn)
constexpr int kFlaggedSlots = 8;

static cudaError_t simt_bwd(const BwdParams& p, const int* flags, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    int P, len;
    simt_segments(p.T, &P, &len);
    const int BH = p.B * p.H;
    const size_t rows = (size_t)BH * p.dk;
    char* w = static_cast<char*>(p.ws);
    float* dqf = reinterpret_cast<float*>(w);
    w += align256(rows * (size_t)p.T * 4);
    float* fin = reinterpret_cast<float*>(w);
    w += align256(rows * 4);
    int* list = nullptr;
    int slots = BH;
    if (flags) {  // the flagged heads, listed on the device
        list = reinterpret_cast<int*>(w);
        w += align256((size_t)(BH + 1) * 4);
        slots = BH < kFlaggedSlots ? BH : kFlaggedSlots;
        simt_flag_list<<<1, 256, 0, s>>>(flags, BH, list);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    SimtSeg sg = {P, len, kSegWhole, nullptr, nullptr, nullptr};
    auto sweep = [&](bool rev) {
        return p.bf16 ? bwd_t<__nv_bfloat16>(p, dqf, fin, list, slots, sg, rev, s)
                      : bwd_t<float>(p, dqf, fin, list, slots, sg, rev, s);
    };
    if (P == 1) {
        cudaError_t e = sweep(false);
        return e != cudaSuccess ? e : sweep(true);
    }
    sg.Sx = reinterpret_cast<float*>(w);
    w += align256(rows * P * (size_t)p.dv * 4);
    sg.La = reinterpret_cast<float*>(w);
    w += align256(rows * P * 4);
    sg.tot = reinterpret_cast<float*>(w);
    const unsigned fgrid = (unsigned)(slots * kFixBlocks);
    cudaError_t e;
    // local maps of sweep F, full passes (each folding the maps before it), the
    // same for sweep R, then the decay-gradient carries
    sg.mode = kSegLocal;
    if ((e = sweep(false)) != cudaSuccess) return e;
    sg.mode = kSegFull;
    if ((e = sweep(false)) != cudaSuccess) return e;
    sg.mode = kSegLocal;
    if ((e = sweep(true)) != cudaSuccess) return e;
    sg.mode = kSegFull;
    if ((e = sweep(true)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(fgrid);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return p.bf16 ? cudaLaunchKernelEx(&cfg, simt_carry_fix<__nv_bfloat16>, p, sg,
                                       static_cast<const float*>(fin), static_cast<const int*>(list), slots)
                  : cudaLaunchKernelEx(&cfg, simt_carry_fix<float>, p, sg, static_cast<const float*>(fin),
                                       static_cast<const int*>(list), slots);
}

cudaError_t launch_simt_bwd(const BwdParams& p, cudaStream_t s) { return simt_bwd(p, nullptr, s); }

cudaError_t launch_simt_bwd_flagged(const BwdParams& p, const int* flags, cudaStream_t s) {
    return simt_bwd(p, flags, s);
}

}  // namespace rdm
