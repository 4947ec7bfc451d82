// quant_weight.cu -- 128x128 block quantization of all experts' weights in one
// launch (Kanana-2 deep dive, devday.kr, FP8 paragraph: one MoE quantization
// kernel instead of one expert after another; DeepSeek-V3 summary sec. 2.2:
// 128x128 weight blocks).
//
// Bound: HBM, 3 bytes per element (2 read, 1 written) + 4 bytes per block.
// One CTA of 256 threads per block, five resident per SM: thread 0 brings the
// whole block (128 rows x 256 bytes) into shared memory with one 2-D TMA load,
// so each SM keeps up to five 32 KB blocks in flight without spending
// registers on them.  The block amax is a 16-bit SIMD max over the staged
// block, a warp shuffle and a shared-memory reduction; each thread then
// converts 8 rows x 8 values (branch-free fast path, exact division only where
// the bracket check asks for it) and writes them as 8-byte stores (a warp
// writes two 128-byte code rows).  (Measured against register-resident blocks
// of 512 threads, two per SM: 0.64 of the copy bandwidth; this one 0.97.)
#include <cuda.h>

#include "fg8_common.cuh"
#include "fg8_tma.cuh"

namespace {

using namespace fg8::tma;

constexpr int kThreads = 256;
constexpr uint32_t kBlockBytes = 128 * 256;   // bf16 128 x 128

__global__ void __launch_bounds__(kThreads, 5)
quant_weight_blocks(const __grid_constant__ CUtensorMap tmW, int64_t N, int64_t K,
                    uint8_t* __restrict__ wq, float* __restrict__ sw, int32_t* status) {
    extern __shared__ __align__(128) uint8_t blk[];   // [128 rows][256 bytes]
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[kThreads / 32];
    __shared__ int abort_flag;
    const int kb = blockIdx.x, nb = blockIdx.y, e = blockIdx.z;
    const int64_t KB = K / 128, NB = N / 128;
    const int t = threadIdx.x;
    const uint32_t b = smem_u32(&bar);
    if (t == 0) {
        abort_flag = 0;
        mbar_init(b, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(b, kBlockBytes);
        tma_load_2d(&tmW, smem_u32(blk), b, kb * 128, (int)(e * N + nb * 128));
    }
    __syncthreads();
    // bounded wait; on a timeout the block's scale becomes NaN (and *status
    // says FG8_ERR_TIMEOUT) rather than a plausible value
    const bool ok = mbar_wait(b, 0, &abort_flag, status);
    const int chunk = t & 15;     // 16-byte chunk of a 256-byte block row
    const int r0 = t >> 4;        // rows r0 + 16 i
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        m = fmaxf(m, fg8::amax8(*reinterpret_cast<const uint4*>(blk + (r0 + 16 * i) * 256 + chunk * 16)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((t & 31) == 0) red[t >> 5] = m;
    __syncthreads();
    float amax = red[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    const float s = fg8::tile_scale(amax);
    const fg8::QScale q = fg8::make_qscale(s);
    const int64_t base = ((int64_t)e * N + (int64_t)nb * 128) * K + (int64_t)kb * 128;
    uint8_t* dst = wq + base + chunk * 8;
#pragma unroll 2
    for (int i = 0; i < 8; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(blk + (r0 + 16 * i) * 256 + chunk * 16);
        *reinterpret_cast<uint2*>(dst + (int64_t)(r0 + 16 * i) * K) = fg8::quant8(v, q);
    }
    if (t == 0) sw[((int64_t)e * NB + nb) * KB + kb] = ok ? s : __int_as_float(0x7FC00000);
}

}  // namespace

extern "C" fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, int32_t* dev_status,
                                          fg8_stream_t stream) {
    if (!w || !wq || !sw) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (N / 128 > 65535 || E > 65535) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(w) || !fg8h::aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3) ||
        (reinterpret_cast<uintptr_t>(dev_status) & 3))
        return FG8_ERR_INVALID_ARG;
    CUtensorMap m;
    if (!fg8h::make_tensor_map_2d(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, (uint64_t)E * N,
                                  (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return FG8_ERR_CUDA;
    if (cudaFuncSetAttribute(quant_weight_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kBlockBytes) != cudaSuccess)
        return FG8_ERR_CUDA;
    dim3 grid(K / 128, N / 128, E);
    quant_weight_blocks<<<grid, kThreads, kBlockBytes, (cudaStream_t)stream>>>(m, N, K, wq, sw,
                                                                               dev_status);
    return fg8h::launch_status();
}
