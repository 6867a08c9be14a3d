// bwd_noalloc.cu -- rdm_ddts_bwd_noalloc: the backward for callers that cannot
// allocate device memory at the point of the call.
//
// The exact CUDA-core backward needs float32 scratch (dq for every token and
// channel, one row per head and, for long sequences, the maps of its sequence
// segments).  rdm_ddts_bwd takes that scratch from the
// caller.  This variant takes it from a fixed array compiled into the library
// instead, so a caller with no allocator at hand -- for example a serving
// process whose device memory was carved up once at start-up and may not grow,
// or a callback that must not call cudaMalloc/cudaFree because those can
// synchronise the whole device -- can still run the backward.
//
// The array is kNoAllocScratchBytes (16 MiB) per device and lives as long as
// the library is loaded.  CUDA loads the library's module on a device lazily,
// so the first call there allocates the array and may synchronise; callers
// make one call at start-up.  The device address is looked up on every call
// (cheap once the module is loaded): nothing cached can go stale across a
// cudaDeviceReset, and no host state is shared between threads.
#include <string.h>

#include "../../include/rdm_ddts.h"
#include "launch.h"

namespace rdm {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code must not hand the symbol itself to a kernel: on the host it names a
// shadow variable, not device memory.  Look up the real address on the current
// device.
rdm_status scratch_for_current_device(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RDM_ERR_CUDA;
    *out = p;
    return RDM_OK;
}

}  // namespace
}  // namespace rdm

extern "C" rdm_status rdm_ddts_bwd_noalloc(const rdm_bwd_args* args, rdm_stream_t stream) {
    if (!args) return RDM_ERR_INVALID_ARG;
    rdm_bwd_args a;
    memcpy(&a, args, sizeof(a));
    a.impl = RDM_IMPL_SIMT;
    a.workspace = nullptr;
    a.workspace_bytes = 0;
    const size_t need = rdm_ddts_bwd_workspace_size(&a);
    if (need == (size_t)-1) return RDM_ERR_INVALID_ARG;
    if (need > rdm::kNoAllocScratchBytes) return RDM_ERR_WORKSPACE;  // problem too large
    if (need > 0) {
        void* scratch = nullptr;
        const rdm_status st = rdm::scratch_for_current_device(&scratch);
        if (st != RDM_OK) return st;
        a.workspace = scratch;
        a.workspace_bytes = rdm::kNoAllocScratchBytes;
    }
    return rdm_ddts_bwd(&a, stream);
}
