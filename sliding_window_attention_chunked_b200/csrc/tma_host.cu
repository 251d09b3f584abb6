// tma_host.cu -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry-point query so that librod.so does not link libcuda).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace rod {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}
}  // namespace

// 3-D tensor [d2][d1][d0] (d0 contiguous) of 2-byte (bf16) or 4-byte (fp32) elements, loaded
// as boxes of box1 rows x box0 elements, zero fill outside the tensor. With swizzle128 the box
// row (box0 * element size) must be exactly 128 bytes; without it, any multiple of 16 bytes.
cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, bool fp32, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint32_t box0, uint32_t box1, bool swizzle128) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const uint64_t es = fp32 ? 4 : 2;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint32_t box0, uint32_t box1) {
    return make_tmap_3d(map, base, false, d0, d1, d2, box0, box1, true);
}

}  // namespace rod
