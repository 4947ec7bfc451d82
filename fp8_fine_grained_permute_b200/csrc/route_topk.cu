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
#include <climits>
#include <cmath>
#include <type_traits>

#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxK = 16;

// (score, index) order of the selection: larger score first, then lower index
FG8_DEV bool better(float a, int ia, float b, int ib) { return a > b || (a == b && ia < ib); }

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
        const float* u = logits + t * E;
        float s[PER_LANE], c[PER_LANE];
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            const int e = lane + 32 * i;
            if (e < E) {
                s[i] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-__ldcs(u + e))));
                c[i] = __fadd_rn(s[i], bl[i]);
            } else {
                s[i] = 0.f;
                c[i] = -INFINITY;
            }
        }
        uint32_t taken = 0;   // bit i: expert lane + 32 i already chosen
        int32_t my_id = -1;   // lane j < k keeps the j-th choice
        float my_s = 0.f;
        for (int j = 0; j < k; ++j) {
            // this lane's best remaining candidate
            float bc = -INFINITY;
            int bi = INT_MAX, bslot = -1;
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) {
                const int e = lane + 32 * i;
                if (e < E && !(taken >> i & 1u) && better(c[i], e, bc, bi)) {
                    bc = c[i];
                    bi = e;
                    bslot = i;
                }
            }
            // warp-wide best
            float wc = bc;
            int wi = bi;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float oc = __shfl_xor_sync(0xffffffffu, wc, off);
                const int oi = __shfl_xor_sync(0xffffffffu, wi, off);
                if (better(oc, oi, wc, wi)) {
                    wc = oc;
                    wi = oi;
                }
            }
            // the owner marks it and hands its affinity to lane j
            float ws = 0.f;
            if (wi == bi && bslot >= 0) {
                taken |= 1u << bslot;
#pragma unroll
                for (int i = 0; i < PER_LANE; ++i)
                    if (i == bslot) ws = s[i];
            }
            ws = __shfl_sync(0xffffffffu, ws, wi & 31);
            if (lane == j) {
                my_id = wi;
                my_s = ws;
            }
        }
        if (lane < k) {
            ids[t * k + lane] = my_id;
            affinity[t * k + lane] = my_s;
        }
    }
}

}  // namespace

extern "C" fg8_status fg8_route_topk(const float* logits, const float* bias, int64_t T, int E,
                                     int k, int32_t* ids, float* affinity, fg8_stream_t stream) {
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > kMaxK || k > E) return FG8_ERR_INVALID_ARG;
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
