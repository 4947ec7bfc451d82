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

}  // namespace fg8h

extern "C" const char* fg8_status_string(fg8_status s) {
    switch (s) {
        case FG8_OK: return "FG8_OK";
        case FG8_ERR_INVALID_ARG: return "FG8_ERR_INVALID_ARG";
        case FG8_ERR_UNSUPPORTED: return "FG8_ERR_UNSUPPORTED";
        case FG8_ERR_CUDA: return "FG8_ERR_CUDA";
        case FG8_ERR_BAD_EXPERT_ID: return "FG8_ERR_BAD_EXPERT_ID";
        case FG8_ERR_TIMEOUT: return "FG8_ERR_TIMEOUT";
    }
    return "FG8_UNKNOWN_STATUS";
}
