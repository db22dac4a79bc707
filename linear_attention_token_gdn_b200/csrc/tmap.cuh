// tmap.cuh -- host-side encoding of the TMA tensor maps the kernels use (through the driver
// entry point cuTensorMapEncodeTiled, looked up once).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace gdn {

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [N, H, D] view of a token-major tensor; box = box_x columns x 1 head x box_z tokens.
inline bool encode_map_3d(CUtensorMap* m, const void* base, int dt, int N, int H, int D, uint32_t box_x,
                          uint32_t box_z, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const int eb = dt == kF32 ? 4 : 2;
    const CUtensorMapDataType t = dt == kF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dt == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N};
    const cuuint64_t strides[2] = {(cuuint64_t)D * eb, (cuuint64_t)H * D * eb};
    const cuuint32_t box[3] = {box_x, 1, box_z};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, t, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdn
