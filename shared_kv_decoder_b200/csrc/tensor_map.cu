// Host-side TMA descriptor encoding for the TMA-fed kernels (prefill, K/V
// projection, decode of bf16 and 8-bit caches).  The driver's cuTensorMapEncodeTiled is reached
// through the runtime's driver entry-point query, so the library links only
// the CUDA runtime.
#include <cuda.h>

#include "launch.h"

namespace yoco {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

bool encode_map_4d(CUtensorMap *m, const void *ptr, bool bytes, bool swizzle128, const uint64_t dims[4],
                   const uint64_t strides_bytes[3], const uint32_t box[4]) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t d[4], s[3];
    cuuint32_t b[4], es[4] = {1, 1, 1, 1};
    for (int i = 0; i < 4; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i < 3; ++i) s[i] = strides_bytes[i];
    return enc(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
               const_cast<void *>(ptr), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16_map_4d(CUtensorMap *m, const void *ptr, const uint64_t dims[4],
                        const uint64_t strides_bytes[3], const uint32_t box[4]) {
    return encode_map_4d(m, ptr, false, true, dims, strides_bytes, box);
}

}  // namespace yoco
