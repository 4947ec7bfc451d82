// quant_weight.cu -- 128x128 block quantization of all experts' weights in one
// launch (Kanana-2 deep dive, devday.kr, FP8 paragraph: one MoE quantization
// kernel instead of one expert after another; DeepSeek-V3 summary sec. 2.2:
// 128x128 weight blocks).
//
// Persistent CTAs of 512 threads; thread t covers the 16-byte chunk (t % 16) of
// rows t/16 + 32 i (i < 4) of a block, 32 bf16 in registers, and prefetches the
// same part of its next block while the current one is reduced and quantized.
// The block amax is a 16-bit SIMD max, a warp shuffle and a shared-memory
// reduction; codes go back as 8-byte stores (a warp writes two 128-byte rows).
// Bound: HBM, 3 bytes per element (2 read, 1 written) + 4 bytes per block.
#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 512;
constexpr int kRowsPerThread = 128 * 16 / kThreads;   // 4 rows of 16 bytes

struct Blocks {
    const uint16_t* w;
    uint8_t* wq;
    float* sw;
    int64_t N, K, KB, NB, nblocks;
};

// first element of block b (blocks ordered e, nb, kb with kb fastest)
__device__ __forceinline__ int64_t block_base(const Blocks& a, int64_t b) {
    const int64_t kb = b % a.KB, rest = b / a.KB;
    const int64_t nb = rest % a.NB, e = rest / a.NB;
    return (e * a.N + nb * 128) * a.K + kb * 128;
}

__device__ __forceinline__ void load_block(const Blocks& a, int64_t base, int chunk, int r0,
                                           uint4 (&v)[kRowsPerThread]) {
    const uint16_t* src = a.w + base + chunk * 8;
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i)
        v[i] = fg8::ld_stream16(src + (int64_t)(r0 + 32 * i) * a.K);
}

// Persistent: each CTA walks blocks blockIdx.x, +gridDim.x, ... and loads the
// next block into registers before reducing and quantizing the current one, so
// every thread always has one block's loads in flight.
__global__ void __launch_bounds__(kThreads)
quant_weight_blocks(const Blocks a) {
    __shared__ float red[2][kThreads / 32];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int chunk = t & 15;     // 16-byte chunk inside a 256-byte block row
    const int r0 = t >> 4;        // rows r0, r0 + 32, r0 + 64, r0 + 96

    uint4 cur[kRowsPerThread], nxt[kRowsPerThread];
    int64_t b = blockIdx.x;
    if (b < a.nblocks) load_block(a, block_base(a, b), chunk, r0, cur);
    for (int it = 0; b < a.nblocks; b += gridDim.x, ++it) {
        const int64_t base = block_base(a, b);
        const int64_t bn = b + gridDim.x;
        if (bn < a.nblocks) load_block(a, block_base(a, bn), chunk, r0, nxt);

        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) m = fmaxf(m, fg8::amax8(cur[i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        float* r = red[it & 1];
        if (lane == 0) r[warp] = m;
        __syncthreads();
        float amax = r[0];
#pragma unroll
        for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, r[i]);

        const float s = fg8::tile_scale(amax);
        const fg8::QScale q = fg8::make_qscale(s);
        uint8_t* dst = a.wq + base + chunk * 8;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i)
            *reinterpret_cast<uint2*>(dst + (int64_t)(r0 + 32 * i) * a.K) = fg8::quant8(cur[i], q);
        if (t == 0) a.sw[b] = s;   // sw[e][nb][kb] is block b
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) cur[i] = nxt[i];
    }
}

}  // namespace

extern "C" fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, fg8_stream_t stream) {
    if (!w || !wq || !sw) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (!fg8h::aligned16(w) || !fg8h::aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3))
        return FG8_ERR_INVALID_ARG;
    Blocks a;
    a.w = w; a.wq = wq; a.sw = sw; a.N = N; a.K = K; a.KB = K / 128; a.NB = N / 128;
    a.nblocks = (int64_t)E * a.NB * a.KB;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_weight_blocks, kThreads, 0) !=
            cudaSuccess || per_sm < 1)
        return FG8_ERR_CUDA;
    int64_t grid = (int64_t)per_sm * fg8h::num_sms();
    if (grid > a.nblocks) grid = a.nblocks;
    quant_weight_blocks<<<(unsigned)grid, kThreads, 0, (cudaStream_t)stream>>>(a);
    return fg8h::launch_status();
}
