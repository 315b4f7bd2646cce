// tc_host.cu -- host-side helpers for the tensor-core kernels: tensor-map
// encoding through the driver entry point (no link-time libcuda dependency).
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace hm {
namespace tc {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    });
    return fn;
}
}  // namespace

bool make_tmap_bf16(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box) {
    return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_tmap(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, int rank,
               const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
               CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5];
    cuuint64_t gstride[4];
    cuuint32_t bdim[5], estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
    }
    for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
    CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstride, bdim, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t ensure_smem_limit_impl(const void *kern, int bytes) {
    struct Entry {
        const void *kern;
        int dev;
        int bytes;
    };
    static std::mutex mu;
    static Entry done[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < n; ++i)
        if (done[i].kern == kern && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && n < 256) done[n++] = Entry{kern, dev, bytes};
    return e;
}

}  // namespace tc
}  // namespace hm
