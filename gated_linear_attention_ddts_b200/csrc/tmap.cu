// tmap.cu -- host construction of TMA tensor maps through the driver entry
// point (no link-time dependency on libcuda), and the small host helpers the
// sequence-segmented launches share (SM count, launch tags).
#include <cudaTypedefs.h>

#include "launch.h"

#include <atomic>
#include <chrono>

namespace rdm {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1,
                       uint64_t n2, uint32_t b0, uint32_t b1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {n0, n1, n2};
    cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d_plain(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1,
                             uint64_t n2, uint32_t b0, uint32_t b1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {n0, n1, n2};
    cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint32_t b0,
                      uint32_t b1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {n0, n1};
    cuuint64_t strides[1] = {n0 * 4};
    cuuint32_t box[2] = {b0, b1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 1;
        cache[dev] = n;
    }
    return cache[dev];
}

unsigned next_launch_tag() {
    static std::atomic<unsigned> counter{
        (unsigned)std::chrono::steady_clock::now().time_since_epoch().count() | 1u};
    const unsigned e = counter.fetch_add(1u) + 1u;
    return e == 0 ? 1u : e;
}

}  // namespace rdm
