// tc_common.cuh -- pieces shared by the tensor-core forward and backward
// kernels: tile geometry, shared-memory operand offsets for the canonical
// no-swizzle UMMA layouts, bf16 pack/unpack and a bounded drain wait.
#pragma once

#include <cuda_bf16.h>

#include "rdm_common.cuh"
#include "tc_ptx.cuh"

namespace rdm {
namespace tc {

constexpr float kSpanMax = 120.0f;              // largest in-window log-decay span
constexpr long long kWaitLimit = 2000000000LL;  // bounded waits: ~1 s of SM clocks
constexpr int kBox = 64 * 64 * 2;               // bytes of one 64x64 bf16 TMA box
// channel-group stride of the Qt / Kt operand tiles: 1024 + 16 bytes, the skew
// spreads the channel groups a warp writes for one token over all banks
constexpr int kQK = 1040;

// ---- shared-memory operand offsets (bytes), canonical no-swizzle UMMA layouts
// A_bf16: K-major, 8-row groups 128 B apart, K groups 1024 B apart
__device__ __forceinline__ uint32_t off_rowmajor64(int r, int k) {
    return (uint32_t)((r >> 3) * 128 + (k >> 3) * 1024 + (r & 7) * 16 + (k & 7) * 2);
}
// Qt, Kt: K-major [token][channel], 8-token groups 128 B apart, channel groups
// kQK B apart
__device__ __forceinline__ uint32_t off_qk(int t, int i) {
    return (uint32_t)((t >> 3) * 128 + (i >> 3) * kQK + (t & 7) * 16 + (i & 7) * 2);
}
// Vh [s][j] stored MN-major for N = j: j groups 1024 B apart, s groups 128 B apart
__device__ __forceinline__ uint32_t off_vh(int s, int j) {
    return (uint32_t)((j >> 3) * 1024 + (s >> 3) * 128 + (s & 7) * 16 + (j & 7) * 2);
}
// S_hat [i][j] stored MN-major for N = j: j groups DK*16 B apart, i groups 128 B apart
template <int DK>
__device__ __forceinline__ uint32_t off_shat(int i, int j) {
    return (uint32_t)((j >> 3) * (DK * 16) + (i >> 3) * 128 + (i & 7) * 16 + (j & 7) * 2);
}
// 8 consecutive bf16 of row t, column group cg, in a tile of 64-wide 128B-swizzled boxes
__device__ __forceinline__ uint32_t off_raw(int t, int cg) {
    return (uint32_t)((cg >> 3) * kBox + t * 128 + (((cg & 7) ^ (t & 7)) << 4));
}

// bf16 -> fp32 is a 16-bit shift of the bit pattern; doing it with integer
// ops keeps it off the conversion pipe that the exp2/log2 instructions need.
__device__ __forceinline__ void unpack8(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    return u;
}

// Element-wise product of two bf16 pairs, rounded once to bf16 (the product of
// two bf16 values is exact in fp32, so this equals widening both, multiplying
// in fp32 and rounding the result: one instruction instead of seven).
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint4 bmul8(uint4 a, uint4 b) {
    return make_uint4(bmul2(a.x, b.x), bmul2(a.y, b.y), bmul2(a.z, b.z), bmul2(a.w, b.w));
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitLimit) return false;
    return true;
}



}  // namespace tc
}  // namespace rdm
