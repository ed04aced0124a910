// tensor_maps.cu -- host-side TMA descriptors shared by the kernels, and the
// device wait limit.
#include <stdlib.h>

#include <string>

#include "internal.h"

namespace veda {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

veda_status encode_tile_map(CUtensorMap* map, const void* base, const Problem& pr,
                            const int* shape) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[5] = {(cuuint64_t)pr.d, (cuuint64_t)pr.Ws, (cuuint64_t)pr.Hs,
                                (cuuint64_t)pr.T, (cuuint64_t)pr.B * pr.H};
    const cuuint64_t strides[4] = {(cuuint64_t)pr.d * 2, (cuuint64_t)pr.Ws * pr.d * 2,
                                   (cuuint64_t)pr.Hs * pr.Ws * pr.d * 2,
                                   (cuuint64_t)pr.N * pr.d * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)shape[2], (cuuint32_t)shape[1],
                               (cuuint32_t)shape[0], 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string((int)r));
    return VEDA_OK;
}

veda_status encode_tile_map_2c(CUtensorMap* map, const void* base, const Problem& pr,
                               const int* shape) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    if (pr.d != 128) return fail(VEDA_ERR_UNSUPPORTED, "two-chunk tile view needs d = 128");
    // (64 channels, x, y, t + T*(b*H + h), channel chunk): the chunk dimension
    // (stride 128 bytes) is the slowest in the box, so one copy lands both
    // 64-channel planes of a tile one after the other
    const cuuint64_t dims[5] = {64, (cuuint64_t)pr.Ws, (cuuint64_t)pr.Hs,
                                (cuuint64_t)pr.T * pr.B * pr.H, 2};
    const cuuint64_t strides[4] = {(cuuint64_t)pr.d * 2, (cuuint64_t)pr.Ws * pr.d * 2,
                                   (cuuint64_t)pr.Hs * pr.Ws * pr.d * 2, 128};
    const cuuint32_t box[5] = {64, (cuuint32_t)shape[2], (cuuint32_t)shape[1],
                               (cuuint32_t)shape[0], 2};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (two-chunk view) failed with code " +
                                       std::to_string((int)r));
    return VEDA_OK;
}

veda_status encode_rows_map(CUtensorMap* map, const float* base, long long rows, int cols,
                            int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed: " + std::to_string((int)r));
    return VEDA_OK;
}

unsigned long long wait_limit_ns() {
    const char* env = getenv("VEDA_WAIT_LIMIT_MS");
    unsigned long long ms = 10000ull;  // a healthy wait takes microseconds
    if (env != nullptr && atoll(env) > 0) ms = (unsigned long long)atoll(env);
    return ms * 1000000ull;
}

}  // namespace veda
