// combine.cu -- unpermute + combine of the experts' output rows.
//
// After the down-projection every routed (token, slot) pair has one output
// row, in expert order.  The layer's output for a token is the sum of its
// pairs' rows weighted by the gate values, the selected sigmoid affinities
// normalized to sum 1 (DeepSeek-V3 summary, sec. 2.1: sigmoid affinity,
// top-K routing; the normalization is the reading stated in fg8.h).
//
// One warp per token: the slot rows and weights are broadcast once, then every
// lane streams 16-byte chunks (8 bf16) of all k rows of the token before
// adding them up, so k loads per lane are in flight at a time; the rows are
// read once (streaming) and each output chunk is written once.
#include <type_traits>

#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxSlots = 16;

FG8_DEV uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// KG: slots unrolled (a power of two >= k), so the row loads of a chunk are
// all issued before the first add and registers are sized for k, not for 16.
template <int KG, bool kF32Out>
__global__ void __launch_bounds__(kThreads)
combine_rows(const uint4* __restrict__ y, const int32_t* __restrict__ token_row,
             const float* __restrict__ affinity, int64_t T, int k, int64_t R, int C8,
             int normalize, void* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; t < T; t += nwarps) {
        // lane j < k holds slot j; rows outside [0, R) are dropped pairs
        int32_t row = -1;
        float a = 0.f;
        if (lane < k) {
            row = token_row[t * k + lane];
            a = affinity[t * k + lane];
            if (row < 0 || (int64_t)row >= R) row = -1;
        }
        // sum of the kept affinities in slot order, then one division each
        float sum = 0.f;
        for (int j = 0; j < k; ++j) {
            const float aj = __shfl_sync(0xffffffffu, a, j);
            const int rj = __shfl_sync(0xffffffffu, row, j);
            if (rj >= 0) sum = __fadd_rn(sum, aj);
        }
        const float w = normalize ? (sum != 0.f ? __fdiv_rn(a, sum) : 0.f) : a;
        int32_t rr[KG];
        float ww[KG];
#pragma unroll
        for (int j = 0; j < KG; ++j) {
            rr[j] = __shfl_sync(0xffffffffu, row, j);
            ww[j] = __shfl_sync(0xffffffffu, w, j);
            if (j >= k) rr[j] = -1;
        }
        for (int c = lane; c < C8; c += 32) {
            uint4 v[KG];
#pragma unroll
            for (int j = 0; j < KG; ++j)
                if (rr[j] >= 0) v[j] = __ldcs(y + (int64_t)rr[j] * C8 + c);
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
            for (int j = 0; j < KG; ++j) {
                if (rr[j] < 0) continue;
                const uint32_t wd[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(ww[j], fg8::bf16_lo(wd[i])));
                    acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(ww[j], fg8::bf16_hi(wd[i])));
                }
            }
            if (kF32Out) {
                float4* o = static_cast<float4*>(out) + (t * C8 + c) * 2;
                __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
                __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
            } else {
                uint4* o = static_cast<uint4*>(out) + t * C8 + c;
                __stcs(o, make_uint4(bf16x2_rn(acc[0], acc[1]), bf16x2_rn(acc[2], acc[3]),
                                     bf16x2_rn(acc[4], acc[5]), bf16x2_rn(acc[6], acc[7])));
            }
        }
    }
}

}  // namespace

extern "C" fg8_status fg8_unpermute_combine(const uint16_t* y, int64_t R, int C,
                                            const int32_t* token_row, const float* affinity,
                                            int64_t T, int k, int normalize, int out_dtype,
                                            void* out, fg8_stream_t stream) {
    if (T < 0 || R < 0 || k < 1 || k > kMaxSlots || C < 8 || C % 8 || (normalize != 0 && normalize != 1))
        return FG8_ERR_INVALID_ARG;
    if (out_dtype != FG8_OUT_BF16 && out_dtype != FG8_OUT_F32) return FG8_ERR_INVALID_ARG;
    if (T == 0) return FG8_OK;
    if (!token_row || !affinity || !out || (R > 0 && !y)) return FG8_ERR_INVALID_ARG;
    if ((R > 0 && !fg8h::aligned16(y)) || !fg8h::aligned16(out) ||
        (reinterpret_cast<uintptr_t>(token_row) & 3) || (reinterpret_cast<uintptr_t>(affinity) & 3))
        return FG8_ERR_INVALID_ARG;
    if (R > INT32_MAX || T > INT64_MAX / k) return FG8_ERR_UNSUPPORTED;
    const int C8 = C / 8;
    const int64_t warps_per_block = kThreads / 32;
    const uint4* yp = reinterpret_cast<const uint4*>(y);
    fg8_status st = FG8_OK;
    auto go = [&](auto kg) {
        constexpr int KG = decltype(kg)::value;
        auto kern = out_dtype == FG8_OUT_F32 ? combine_rows<KG, true> : combine_rows<KG, false>;
        // one wave: the blocks that fit on every SM at once, token loop inside
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess ||
            per_sm < 1) {
            st = FG8_ERR_CUDA;
            return;
        }
        int64_t grid = (T + warps_per_block - 1) / warps_per_block;
        const int64_t cap = (int64_t)fg8h::num_sms() * per_sm;
        if (grid > cap) grid = cap;
        kern<<<(unsigned)grid, kThreads, 0, (cudaStream_t)stream>>>(yp, token_row, affinity, T, k, R,
                                                                   C8, normalize, out);
        st = fg8h::launch_status();
    };
    if (k <= 2) go(std::integral_constant<int, 2>());
    else if (k <= 4) go(std::integral_constant<int, 4>());
    else if (k <= 8) go(std::integral_constant<int, 8>());
    else go(std::integral_constant<int, 16>());
    return st;
}
