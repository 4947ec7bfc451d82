// quant_weight.cu -- 128x128 block quantization of all experts' weights in one
// launch (Kanana-2 deep dive, devday.kr, FP8 paragraph: one MoE quantization
// kernel instead of one expert after another; DeepSeek-V3 summary sec. 2.2:
// 128x128 weight blocks).
//
// Bound: HBM, 3 bytes per element (2 read, 1 written) + 4 bytes per block.
// To keep enough bytes in flight, each SM runs one persistent CTA that streams
// its blocks (b = blockIdx.x, +gridDim.x, ...) through a ring of kStages
// shared-memory stages filled by 2-D TMA loads (128 rows x 256 bytes, 32 KB),
// so kStages blocks are always in flight regardless of registers.  Per block:
//   all threads wait for the stage (bounded), read their 4 x 16 bytes, and
//   reduce the amax (16-bit SIMD max -> warp shuffle -> shared memory);
//   thread 0 refills the stage with the block kStages ahead;
//   every thread quantizes its 32 values into a shared code buffer, and
//   thread 0 writes the 128 x 128-byte code block back with a TMA store
//   (two code buffers, so a store overlaps the next block).
#include "fg8_common.cuh"
#include "fg8_tma.cuh"

namespace {

using namespace fg8::tma;

constexpr int kThreads = 512;
constexpr int kStages = 5;
constexpr uint32_t kInBytes = 128 * 128 * 2;      // one bf16 block
constexpr uint32_t kOutBytes = 128 * 128;         // one code block
constexpr int kOutBufs = 2;
constexpr uint32_t kOffOut = kStages * kInBytes;                  // 163840
constexpr uint32_t kOffBars = kOffOut + kOutBufs * kOutBytes;      // 196608
constexpr uint32_t kOffRed = kOffBars + 8 * kStages;
constexpr uint32_t kSmem = kOffRed + 2 * 4 * (kThreads / 32) + 1024;   // + alignment slack
static_assert(kSmem <= 232448, "shared memory per CTA");

__global__ void __launch_bounds__(kThreads, 1)
quant_weight_tma(const __grid_constant__ CUtensorMap tin, const __grid_constant__ CUtensorMap tout,
                 float* __restrict__ sw, int64_t nblocks, int64_t KB, int32_t* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    float* red = reinterpret_cast<float*>(smem + kOffRed);   // [2][16]
    __shared__ int s_abort;

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int chunk = t & 15;     // 16-byte chunk of a 256-byte block row
    const int r0 = t >> 4;        // rows r0 + 32 i, i < 4
    const int64_t G = gridDim.x;

    auto full_bar = [&](int s) { return sbase + kOffBars + 8u * s; };
    // block b -> (x = first column, y = first row of the [E*N][K] matrix)
    auto coords = [&](int64_t b, int& x, int& y) {
        x = (int)((b % KB) * 128);
        y = (int)((b / KB) * 128);
    };

    if (t == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(full_bar(s), 1);
        s_abort = 0;
        fence_barrier_init();
        for (int s = 0; s < kStages; ++s) {
            const int64_t b = blockIdx.x + s * G;
            if (b < nblocks) {
                int x, y;
                coords(b, x, y);
                mbar_arrive_expect_tx(full_bar(s), kInBytes);
                tma_load_2d(&tin, sbase + s * kInBytes, full_bar(s), x, y);
            }
        }
    }
    __syncthreads();

    for (int64_t it = 0;; ++it) {
        const int64_t b = blockIdx.x + it * G;
        if (b >= nblocks) break;
        const int s = (int)(it % kStages);
        const uint32_t parity = (uint32_t)((it / kStages) & 1);
        const bool ok = mbar_wait(full_bar(s), parity, &s_abort, status);
        if (__syncthreads_or(!ok)) break;

        const uint8_t* in = smem + s * kInBytes;
        uint4 v[4];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i] = *reinterpret_cast<const uint4*>(in + (r0 + 32 * i) * 256 + chunk * 16);
            m = fmaxf(m, fg8::amax8(v[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        float* rb = red + (it & 1) * (kThreads / 32);
        if (lane == 0) rb[warp] = m;
        const int ob = (int)(it & 1);
        // the store that last used this code buffer (two blocks ago) must have
        // finished reading it before anyone writes it again
        if (t == 0) bulk_wait_read<kOutBufs - 1>();
        __syncthreads();

        // every thread has its data: refill this stage with the block kStages ahead
        if (t == 0) {
            const int64_t bn = b + kStages * G;
            if (bn < nblocks) {
                int x, y;
                coords(bn, x, y);
                mbar_arrive_expect_tx(full_bar(s), kInBytes);
                tma_load_2d(&tin, sbase + s * kInBytes, full_bar(s), x, y);
            }
        }
        float amax = rb[0];
#pragma unroll
        for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, rb[i]);
        const float sc = fg8::tile_scale(amax);
        const fg8::QScale q = fg8::make_qscale(sc);
        uint8_t* out = smem + kOffOut + ob * kOutBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint2*>(out + (r0 + 32 * i) * 128 + chunk * 8) = fg8::quant8(v[i], q);
        fence_async_shared();
        __syncthreads();
        if (t == 0) {
            int x, y;
            coords(b, x, y);
            tma_store_2d(&tout, sbase + kOffOut + ob * kOutBytes, x, y);
            bulk_commit();
            sw[b] = sc;   // sw[e][nb][kb] is block b
        }
    }
    if (t == 0) bulk_wait_all();
}

}  // namespace

extern "C" fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, fg8_stream_t stream) {
    if (!w || !wq || !sw) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (!fg8h::aligned16(w) || !fg8h::aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3))
        return FG8_ERR_INVALID_ARG;
    const uint64_t rows = (uint64_t)E * N;
    if (rows > 0xFFFFFFFFull) return FG8_ERR_UNSUPPORTED;
    CUtensorMap tin, tout;
    if (!fg8h::make_tensor_map_2d(&tin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, rows, K, 128, 128,
                                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !fg8h::make_tensor_map_2d(&tout, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, rows, K, 128, 128,
                                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return FG8_ERR_CUDA;
    const int64_t KB = K / 128;
    const int64_t nblocks = (int64_t)E * (N / 128) * KB;
    if (cudaFuncSetAttribute(quant_weight_tma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmem) != cudaSuccess)
        return FG8_ERR_CUDA;
    int64_t grid = fg8h::num_sms();
    if (grid > nblocks) grid = nblocks;
    quant_weight_tma<<<(unsigned)grid, kThreads, kSmem, (cudaStream_t)stream>>>(
        tin, tout, sw, nblocks, KB, nullptr);
    return fg8h::launch_status();
}
