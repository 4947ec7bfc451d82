// route_topk.cu -- sigmoid-affinity top-K routing with a per-expert bias.
//
// DeepSeek-V3 summary, sec. 2.1: each token's affinity to an expert is a
// sigmoid score; the K experts with the largest scores are chosen, and a
// per-expert bias, adjusted to balance the load, enters the choice (not the
// gate values).  Here: s = sigmoid(u), the choice ranks s + bias, the
// affinities written out are s of the chosen experts (the combine normalizes
// them).
//
// One warp per token: lane l holds experts l, l + 32, ... in registers; K
// rounds of a warp-wide (score, index) max pick the experts in descending
// order, ties to the lower index.
#include <type_traits>

#include "fg8_common.cuh"
#include "fg8_route.cuh"

namespace {

constexpr int kThreads = 256;

template <int PER_LANE>
__global__ void __launch_bounds__(kThreads)
route_topk_rows(const float* __restrict__ logits, const float* __restrict__ bias, int64_t T, int E,
                int k, int32_t* __restrict__ ids, float* __restrict__ affinity) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    float bl[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        bl[i] = e < E ? bias[e] : 0.f;
    }
    for (int64_t t = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; t < T; t += nwarps) {
        int32_t my_id;
        float my_s;
        fg8::route_token<PER_LANE>(logits + t * E, bl, E, k, lane, my_id, my_s);
        if (lane < k) {
            ids[t * k + lane] = my_id;
            affinity[t * k + lane] = my_s;
        }
    }
}

}  // namespace

extern "C" fg8_status fg8_route_topk(const float* logits, const float* bias, int64_t T, int E,
                                     int k, int32_t* ids, float* affinity, fg8_stream_t stream) {
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > fg8::kRouteMaxK || k > E) return FG8_ERR_INVALID_ARG;
    if (T == 0) return FG8_OK;
    if (!logits || !bias || !ids || !affinity) return FG8_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(bias) |
         reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(affinity)) & 3)
        return FG8_ERR_INVALID_ARG;
    if (T > INT64_MAX / E) return FG8_ERR_UNSUPPORTED;
    fg8_status st = FG8_OK;
    auto go = [&](auto pl) {
        constexpr int PL = decltype(pl)::value;
        auto kern = route_topk_rows<PL>;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess ||
            per_sm < 1) {
            st = FG8_ERR_CUDA;
            return;
        }
        int64_t grid = (T + kThreads / 32 - 1) / (kThreads / 32);
        const int64_t cap = (int64_t)fg8h::num_sms() * per_sm;
        if (grid > cap) grid = cap;
        kern<<<(unsigned)grid, kThreads, 0, (cudaStream_t)stream>>>(logits, bias, T, E, k, ids,
                                                                   affinity);
        st = fg8h::launch_status();
    };
    if (E <= 64) go(std::integral_constant<int, 2>());
    else if (E <= 128) go(std::integral_constant<int, 4>());
    else if (E <= 256) go(std::integral_constant<int, 8>());
    else if (E <= 512) go(std::integral_constant<int, 16>());
    else go(std::integral_constant<int, 32>());
    return st;
}
