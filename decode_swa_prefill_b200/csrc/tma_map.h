// Host-side TMA tensor maps for the [B,T,H,d] bf16 tensors of the tcgen05
// kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

namespace swa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); null when the driver does not provide it.
inline EncodeTiledFn get_encode()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B,T,H,d] bf16 viewed as the 4-D tensor (d, H, T, B); box = one swizzle
// chunk of `rows` rows of one head: min(d, 64) elements per row, 128-byte
// swizzle for 64-element rows, 64-byte swizzle for 32-element rows.  Boxes
// that reach outside the tensor (rows before 0 or past T) read zeros.
inline bool make_bthd_map(CUtensorMap *m, const void *ptr, int B, int T, int H, int d, int rows)
{
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const int e = d * 2 >= 128 ? 64 : d; // elements per swizzled row
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    cuuint32_t box[4] = {(cuuint32_t)e, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, e == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace swa
