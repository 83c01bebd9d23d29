// gdn_tma.cu -- tensor maps (TMA descriptors) of the prefill kernels.  The
// driver's encoder is reached through cudaGetDriverEntryPoint, so the library
// links against the CUDA runtime only and loads on machines without a GPU.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [tokens, heads] fp32 gates viewed as 2-D, boxes of 4 heads x 64 tokens (the
// inner box must span at least 16 bytes; the kernel picks its head's column).
bool make_gate_map(CUtensorMap *map, const float *base, int heads, int tokens) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(heads), cuuint64_t(tokens)};
    const cuuint64_t strides[1] = {cuuint64_t(heads) * 4};
    const cuuint32_t box[2] = {4, 64};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [tokens, heads, 128] bf16 viewed as a 3-D tensor (d fastest), boxes of
// 64 (d) x 1 (head) x 64 (tokens), 128-byte swizzle; rows past the last token
// read as zeros.  With `out` set: boxes of 128 (d) x 1 x 64 tokens, no
// swizzle -- the token-major output tile staged in shared memory.
bool make_map(CUtensorMap *map, const void *base, int heads, int tokens, bool out) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, cuuint64_t(heads), cuuint64_t(tokens)};
    const cuuint64_t strides[2] = {128 * 2, cuuint64_t(heads) * 128 * 2};
    const cuuint32_t box[3] = {out ? 128u : 64u, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, out ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `rows` x 64 bf16 matrix (rows of 128 bytes) in boxes of 64 rows, 128-byte
// swizzle: the 64 x 64 tiles of the chunk inverses.
bool make_tile_map(CUtensorMap *map, const void *base, int64_t rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {64, cuuint64_t(rows)};
    const cuuint64_t strides[1] = {64 * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdn
