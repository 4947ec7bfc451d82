// api.cu -- host-side pieces of the C ABI shared by all entry points.
#include "fg8_common.cuh"

namespace fg8h {

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        n = 1;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes,
                        const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fg8h

extern "C" const char* fg8_status_string(fg8_status s) {
    switch (s) {
        case FG8_OK: return "FG8_OK";
        case FG8_ERR_INVALID_ARG: return "FG8_ERR_INVALID_ARG";
        case FG8_ERR_UNSUPPORTED: return "FG8_ERR_UNSUPPORTED";
        case FG8_ERR_CUDA: return "FG8_ERR_CUDA";
        case FG8_ERR_BAD_EXPERT_ID: return "FG8_ERR_BAD_EXPERT_ID";
        case FG8_ERR_TIMEOUT: return "FG8_ERR_TIMEOUT";
        case FG8_ERR_WORKSPACE_SHARED: return "FG8_ERR_WORKSPACE_SHARED";
    }
    return "FG8_UNKNOWN_STATUS";
}
