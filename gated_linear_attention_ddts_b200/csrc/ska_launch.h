// ska_launch.h -- host launchers of the sliding-window shared-key attention
// (ska.cu) behind the C ABI, and the device status bit its decode sets.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace rdm {

// Device status word bit: a value read on the device was out of range (a
// negative decode position).  kErrTimeout (rdm_common.cuh) is bit 0.
constexpr unsigned kErrBadValue = 2u;

// Sliding-window shared-key attention (ska.cu), bf16 only.
struct SkaParams {
    int B, H, T, dk, dv, window;
    float scale;           // score scale (> 0)
    const void *q, *k, *v; // q [B,H,T,dk], k [B,T,dk] (shared by the heads), v [B,H,T,dv]
    void* o;               // [B,H,T,dv]
    void* k_cache;         // [B,window,dk] ring filled after the forward, or null
    void* v_cache;         // [B,H,window,dv] ring, or null
    int* pos;              // [B] set to T after the forward, or null
    unsigned* err;
    long long wait_limit;
    int withhold;          // test hook: the producer never loads value tiles
};
struct SkaDecodeParams {
    int B, H, dk, dv, window;
    float scale;
    const void *q, *k, *v; // q [B,H,dk], k [B,dk], v [B,H,dv]
    void* k_cache;         // [B,window,dk]
    void* v_cache;         // [B,H,window,dv]
    int* pos;              // [B] tokens before this one
    int advance;           // add one to pos after the step
    void* o;               // [B,H,dv]
    unsigned* err;         // device status word (a negative position sets kErrBadValue)
};
cudaError_t launch_ska_fwd(const SkaParams& p, cudaStream_t s);
cudaError_t launch_ska_decode(const SkaDecodeParams& p, cudaStream_t s);

}  // namespace rdm
