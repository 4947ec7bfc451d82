// quant_weight.cu -- 128x128 block quantization of all experts' weights in one
// launch (Kanana-2 deep dive, devday.kr, FP8 paragraph: one MoE quantization
// kernel instead of one expert after another; DeepSeek-V3 summary sec. 2.2:
// 128x128 weight blocks).
//
// One CTA per block: 256 threads, thread t covers the 16-byte chunk (t % 16) of
// rows t/16, t/16 + 16, ..., i.e. 8 x 16 B = 64 bf16 held in registers.  All
// loads are issued before any use (64 KB in flight per 8 CTAs), the block
// amax is a warp-shuffle + shared-memory reduction, and each thread writes its
// codes back as 8-byte stores (a warp writes two full 128-byte code rows).
// Bound: HBM, 3 bytes per element (2 read, 1 written) + 4 bytes per block.
#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
quant_weight_blocks(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                    uint8_t* __restrict__ wq, float* __restrict__ sw) {
    const int kb = blockIdx.x, nb = blockIdx.y, e = blockIdx.z;
    const int64_t KB = K / 128, NB = N / 128;
    const int t = threadIdx.x;
    const int chunk = t & 15;     // 16-byte chunk inside a 256-byte row
    const int r0 = t >> 4;        // first row of this thread

    const int64_t base = ((int64_t)e * N + (int64_t)nb * 128) * K + (int64_t)kb * 128;
    const uint16_t* src = w + base + chunk * 8;

    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fg8::ld_stream16(src + (int64_t)(r0 + 16 * i) * K);

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fg8::amax8(v[i]));
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

    uint8_t* dst = wq + base + chunk * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint2*>(dst + (int64_t)(r0 + 16 * i) * K) = fg8::quant8(v[i], q);

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
