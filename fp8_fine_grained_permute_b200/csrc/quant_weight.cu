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
// converts 8 rows x 8 values with the branch-free fast path and writes them as
// 8-byte stores (a warp writes two 128-byte code rows); the groups whose
// bracket check failed are redone exactly after that loop, shared out over the
// warp.  (Measured against register-resident blocks of 512 threads, two per
// SM: 0.64 of the copy bandwidth; this one 0.97.)
#include <cuda.h>

#include "fg8_common.cuh"
#include "fg8_tma.cuh"

namespace {

using namespace fg8::tma;

constexpr int kThreads = 256;
constexpr uint32_t kBlockBytes = 128 * 256;   // bf16 128 x 128
constexpr int kFixCap = 64;                    // failed groups a warp redoes together

// word w of code row r sits at word w ^ swz(r) of the shared code tile: conflict
// free both for the row-wise writes and for the transposed reads below
__device__ __forceinline__ int swz(int r) { return ((r >> 2) ^ (r & 3)) & 31; }

// kT: also write the block-transposed copy (wqT[e][k][n] = wq[e][n][k],
// swT[e][kb][nb] = sw[e][nb][kb]) from the codes still in shared memory, so
// the backward pass's copy costs no second read of wq.
template <bool kT>
__global__ void __launch_bounds__(kThreads, 5)
quant_weight_blocks(const __grid_constant__ CUtensorMap tmW, const uint16_t* __restrict__ w, int64_t N, int64_t K,
                    uint8_t* __restrict__ wq, float* __restrict__ sw, uint8_t* __restrict__ wqT,
                    float* __restrict__ swT, int32_t* status) {
    extern __shared__ __align__(128) uint8_t blk[];   // [128 rows][256 bytes]
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[kThreads / 32];
    __shared__ uint16_t fix_list[kThreads / 32][kFixCap];
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
    // kT: code row r (128 bytes) goes into the first half of bf16 row r's own
    // bytes.  Row r is read only by the 16 lanes that write its codes (two
    // rows per warp), so a warp barrier between the reads and the writes is
    // enough, and no second tile is needed.
    uint32_t* codes = reinterpret_cast<uint32_t*>(blk);   // row r at word 64 r
    // Groups whose fast path failed are only recorded here (bit i) and redone
    // after the loop, so the loop stays branch-free (a few groups in a hundred
    // fail, mostly values that land exactly on a rounding midpoint).
    uint32_t redo = 0;
#pragma unroll 2
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + 16 * i;
        const uint4 v = *reinterpret_cast<const uint4*>(blk + r * 256 + chunk * 16);
        uint2 c, h;
        fg8::quant8_bracket(v, q, c, h);
        redo |= (uint32_t)(q.exact || !fg8::bracket_agrees(c, h)) << i;
        *reinterpret_cast<uint2*>(dst + (int64_t)r * K) = c;
        if (kT) {
            __syncwarp();
            codes[r * 64 + ((2 * chunk) ^ swz(r))] = c.x;
            codes[r * 64 + ((2 * chunk + 1) ^ swz(r))] = c.y;
        }
    }
    // exact codes of those groups over the fast-path ones, shared out over the
    // warp (the staged row may already hold codes, so the values come from
    // global memory; the fast-path stores were made before the warp barrier)
    const int warp = t >> 5;
    auto redo_group = [&](int owner, int i) {
        const int to = 32 * warp + owner;
        const int ch = to & 15, r = (to >> 4) + 16 * i;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(
            w + (((int64_t)e * N + (int64_t)nb * 128 + r) * K + (int64_t)kb * 128 + ch * 8)));
        const uint2 c = fg8::quant8_redo(v, q);
        *reinterpret_cast<uint2*>(wq + base + ch * 8 + (int64_t)r * K) = c;
        if (kT) {
            codes[r * 64 + ((2 * ch) ^ swz(r))] = c.x;
            codes[r * 64 + ((2 * ch + 1) ^ swz(r))] = c.y;
        }
    };
    if (!fg8::coop_redo(redo, fix_list[warp], kFixCap, redo_group)) {
        while (redo != 0u) {
            const int i = __ffs(redo) - 1;
            redo &= redo - 1u;
            redo_group(t & 31, i);
        }
    }
    const float s_out = ok ? s : __int_as_float(0x7FC00000);
    if (t == 0) sw[((int64_t)e * NB + nb) * KB + kb] = s_out;
    if (kT) {
        __syncthreads();
        // lane i of the warp on word column j reads words j of code rows
        // 4i..4i+3, transposes the 4x4 bytes and writes word i of output rows
        // 4j..4j+3: each warp store is one 128-byte output row segment
        const int lane = t & 31, warp = t >> 5;
        uint8_t* dT = wqT + ((int64_t)e * K + (int64_t)kb * 128) * N + (int64_t)nb * 128;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = warp + 8 * jj;
            const uint32_t a0 = codes[(4 * lane + 0) * 64 + (j ^ swz(4 * lane + 0))];
            const uint32_t a1 = codes[(4 * lane + 1) * 64 + (j ^ swz(4 * lane + 1))];
            const uint32_t a2 = codes[(4 * lane + 2) * 64 + (j ^ swz(4 * lane + 2))];
            const uint32_t a3 = codes[(4 * lane + 3) * 64 + (j ^ swz(4 * lane + 3))];
            const uint32_t t0 = __byte_perm(a0, a1, 0x5140), t1 = __byte_perm(a2, a3, 0x5140);
            const uint32_t t2 = __byte_perm(a0, a1, 0x7362), t3 = __byte_perm(a2, a3, 0x7362);
            uint32_t* d = reinterpret_cast<uint32_t*>(dT + (int64_t)(4 * j) * N) + lane;
            d[0] = __byte_perm(t0, t1, 0x5410);
            d[N / 4] = __byte_perm(t0, t1, 0x7632);
            d[2 * (N / 4)] = __byte_perm(t2, t3, 0x5410);
            d[3 * (N / 4)] = __byte_perm(t2, t3, 0x7632);
        }
        if (t == 0) swT[((int64_t)e * KB + kb) * NB + nb] = s_out;
    }
}

fg8_status launch(const uint16_t* w, int E, int N, int K, uint8_t* wq, float* sw, uint8_t* wqT,
                  float* swT, int32_t* dev_status, cudaStream_t stream) {
    if (!w || !wq || !sw) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (N / 128 > 65535 || E > 65535) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(w) || !fg8h::aligned16(wq) || (reinterpret_cast<uintptr_t>(sw) & 3) ||
        (reinterpret_cast<uintptr_t>(dev_status) & 3))
        return FG8_ERR_INVALID_ARG;
    const bool tr = wqT != nullptr;
    if (tr && (!swT || !fg8h::aligned16(wqT) || (reinterpret_cast<uintptr_t>(swT) & 3)))
        return FG8_ERR_INVALID_ARG;
    CUtensorMap m;
    if (!fg8h::make_tensor_map_2d(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, (uint64_t)E * N,
                                  (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return FG8_ERR_CUDA;
    auto kern = tr ? quant_weight_blocks<true> : quant_weight_blocks<false>;
    const uint32_t smem = kBlockBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FG8_ERR_CUDA;
    dim3 grid(K / 128, N / 128, E);
    kern<<<grid, kThreads, smem, stream>>>(m, w, N, K, wq, sw, wqT, swT, dev_status);
    return fg8h::launch_status();
}

}  // namespace

extern "C" fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, int32_t* dev_status,
                                          fg8_stream_t stream) {
    return launch(w, E, N, K, wq, sw, nullptr, nullptr, dev_status, (cudaStream_t)stream);
}

extern "C" fg8_status fg8_quantize_weight_transposed(const uint16_t* w, int E, int N, int K,
                                                     uint8_t* wq, float* sw, uint8_t* wqT,
                                                     float* swT, int32_t* dev_status,
                                                     fg8_stream_t stream) {
    if (!wqT || !swT) return FG8_ERR_INVALID_ARG;
    return launch(w, E, N, K, wq, sw, wqT, swT, dev_status, (cudaStream_t)stream);
}
