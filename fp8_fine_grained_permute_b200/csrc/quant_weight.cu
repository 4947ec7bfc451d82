// quant_weight.cu -- 128x128 block quantization of all experts' weights in one
// launch (Kanana-2 deep dive, devday.kr, FP8 paragraph: one MoE quantization
// kernel instead of one expert after another; DeepSeek-V3 summary sec. 2.2:
// 128x128 weight blocks).
//
// Bound: HBM, 3 bytes per element (2 read, 1 written) + 4 bytes per block.
// One CTA of 512 threads per block, two resident per SM (64 registers): thread
// t loads the 16-byte chunk (t % 16) of rows t/16 + 32 i (i < 4) -- all four
// loads issued before any use -- so each SM keeps two whole blocks (64 KB) in
// flight while another pair computes.  The block amax is a 16-bit SIMD max,
// a warp shuffle and a shared-memory reduction; the 32 values of a thread are
// converted with the branch-free fast path and one combined exactness check;
// codes leave as 8-byte stores (a warp writes two 128-byte code rows).
// (Measured against a persistent version that streams blocks through a TMA
// ring into shared memory: that one serialises each block's compute behind
// CTA-wide barriers with one CTA per SM and ran ~20 % slower.)
#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 512;
constexpr int kPer = 128 * 16 / kThreads;   // 16-byte pieces per thread (4)

__global__ void __launch_bounds__(kThreads, 2)
quant_weight_blocks(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                    uint8_t* __restrict__ wq, float* __restrict__ sw) {
    const int kb = blockIdx.x, nb = blockIdx.y, e = blockIdx.z;
    const int64_t KB = K / 128, NB = N / 128;
    const int t = threadIdx.x;
    const int chunk = t & 15;     // 16-byte chunk inside a 256-byte block row
    const int r0 = t >> 4;        // rows r0 + 32 i

    const int64_t base = ((int64_t)e * N + (int64_t)nb * 128) * K + (int64_t)kb * 128;
    const uint16_t* src = w + base + chunk * 8;
    uint4 v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) v[i] = fg8::ld_stream16(src + (int64_t)(r0 + 32 * i) * K);

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) m = fmaxf(m, fg8::amax8(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float red[kThreads / 32];
    if ((t & 31) == 0) red[t >> 5] = m;
    __syncthreads();
    float amax = red[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, red[i]);

    const float s = fg8::tile_scale(amax);
    const fg8::QScale q = fg8::make_qscale(s);
    uint2 c[kPer];
    fg8::quant8xN<kPer>(v, q, c);
    uint8_t* dst = wq + base + chunk * 8;
#pragma unroll
    for (int i = 0; i < kPer; ++i) *reinterpret_cast<uint2*>(dst + (int64_t)(r0 + 32 * i) * K) = c[i];
    if (t == 0) sw[((int64_t)e * NB + nb) * KB + kb] = s;
}

}  // namespace

extern "C" fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, fg8_stream_t stream) {
    if (!w || !wq || !sw) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (N / 128 > 65535 || E > 65535) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(w) || !fg8h::aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3))
        return FG8_ERR_INVALID_ARG;
    dim3 grid(K / 128, N / 128, E);
    quant_weight_blocks<<<grid, kThreads, 0, (cudaStream_t)stream>>>(w, N, K, wq, sw);
    return fg8h::launch_status();
}
