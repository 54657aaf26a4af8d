// tmap_host.h -- host-side construction of TMA tensor maps (CUtensorMap) for the
// sm_100a kernels. The driver's encoder is fetched once through the runtime's
// driver-entry-point query, so the library does not link libcuda directly.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ab {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tmap_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D bf16 map: extents (x, y, z) with x contiguous, byte strides of y and z, box
// box_x x box_y x 1 with 128-byte swizzle (box_x * 2 must be 128). Elements outside
// the extents read as zero.
inline bool make_tmap_bf16_3d(CUtensorMap *tm, const void *base, uint64_t x, uint64_t y,
                              uint64_t z, uint64_t y_stride, uint64_t z_stride, uint32_t box_x,
                              uint32_t box_y)
{
    EncodeTiledFn enc = tmap_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {x, y, z};
    const cuuint64_t strides[2] = {y_stride, z_stride};
    const cuuint32_t box[3] = {box_x, box_y, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ab
