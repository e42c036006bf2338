// Host-side helpers: TMA tensor maps for the token-major [B*T, H, channels] tensors, and the
// once-per-device dynamic shared-memory opt-in of the kernels.
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "carve_mma.cuh"

namespace carve {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

cudaError_t make_token_tile_map(CUtensorMap *map, const void *base, int elem_bytes, int inner, int H,
                                long long rows, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)inner * elem_bytes, (cuuint64_t)inner * elem_bytes * H};
    const cuuint32_t box[3] = {(cuuint32_t)inner, 1u, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = enc(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The opt-in above 48 KB of dynamic shared memory is a per-device attribute of the kernel that
// persists, so it is set on the first launch on each device only (launches stay one driver
// call; safe to call from several threads).
cudaError_t set_smem_once(const void *kern, int bytes) {
    struct Entry {
        const void *kern;
        int dev, bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &x : done)
        if (x.kern == kern && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.push_back(Entry{kern, dev, bytes});
    return e;
}

}  // namespace carve
