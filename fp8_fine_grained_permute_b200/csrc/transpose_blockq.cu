// transpose_blockq.cu -- transpose of a block-quantized FP8 weight and of its
// scale grid, for the backward pass, so that only the forward FP8 weight needs
// to be stored (Kanana-2 deep dive, devday.kr, FP8 paragraph, last sentence).
//
// wqT[e][k][n] = wq[e][n][k],  swT[e][kb][nb] = sw[e][nb][kb].  No arithmetic:
// the blocks are square, so the scales travel with their blocks unchanged.
//
// One CTA per 128x128 byte block (16 KB), staged through shared memory:
//  1. 16-byte coalesced loads; each word w of row r is stored at word
//     (w ^ f(r)) of shared row r, f(r) = (r >> 2) ^ (r & 3).  A warp stores
//     rows 4a..4a+3, 8 chunks each: the XOR spreads those 32 words over 32
//     banks.
//  2. Lane i of the warp handling word column j reads words j of rows
//     4i..4i+3 (banks j ^ i ^ m: conflict-free), transposes the 4x4 byte block
//     with byte permutes, and writes word i of output rows 4j..4j+3: each
//     warp store is one contiguous 128-byte output row segment.
// Bound: HBM, 2 bytes per element (1 read + 1 written) + 8 bytes per block.
#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int swz(int r) { return ((r >> 2) ^ (r & 3)) & 31; }

__global__ void __launch_bounds__(kThreads)
transpose_blocks(const uint8_t* __restrict__ wq, const float* __restrict__ sw,
                 int64_t N, int64_t K, uint8_t* __restrict__ wqT, float* __restrict__ swT) {
    __shared__ uint32_t tile[128 * 32];
    const int kb = blockIdx.x, nb = blockIdx.y, e = blockIdx.z;
    const int64_t KB = K / 128, NB = N / 128;
    const int t = threadIdx.x;

    const uint8_t* src = wq + ((int64_t)e * N + (int64_t)nb * 128) * K + (int64_t)kb * 128;
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int idx = t + kThreads * i;       // 1024 chunks of 16 bytes
        int r = idx >> 3, c = idx & 7;
        v[i] = fg8::ld_stream16(src + (int64_t)r * K + c * 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int idx = t + kThreads * i;
        int r = idx >> 3, c = idx & 7;
        int f = swz(r);
        uint32_t* row = tile + r * 32;
        row[(4 * c + 0) ^ f] = v[i].x;
        row[(4 * c + 1) ^ f] = v[i].y;
        row[(4 * c + 2) ^ f] = v[i].z;
        row[(4 * c + 3) ^ f] = v[i].w;
    }
    __syncthreads();

    const int lane = t & 31, warp = t >> 5;
    uint8_t* dst = wqT + ((int64_t)e * K + (int64_t)kb * 128) * N + (int64_t)nb * 128;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int j = warp + 8 * jj;      // word column of the input = output row group
        const int i = lane;               // input row group = output word
        uint32_t a0 = tile[(4 * i + 0) * 32 + (j ^ swz(4 * i + 0))];
        uint32_t a1 = tile[(4 * i + 1) * 32 + (j ^ swz(4 * i + 1))];
        uint32_t a2 = tile[(4 * i + 2) * 32 + (j ^ swz(4 * i + 2))];
        uint32_t a3 = tile[(4 * i + 3) * 32 + (j ^ swz(4 * i + 3))];
        // byte c of a_m is element (row 4i+m, col 4j+c); output word for row
        // 4j+c holds bytes (a0.c, a1.c, a2.c, a3.c)
        uint32_t t0 = __byte_perm(a0, a1, 0x5140);
        uint32_t t1 = __byte_perm(a2, a3, 0x5140);
        uint32_t t2 = __byte_perm(a0, a1, 0x7362);
        uint32_t t3 = __byte_perm(a2, a3, 0x7362);
        uint32_t o0 = __byte_perm(t0, t1, 0x5410);
        uint32_t o1 = __byte_perm(t0, t1, 0x7632);
        uint32_t o2 = __byte_perm(t2, t3, 0x5410);
        uint32_t o3 = __byte_perm(t2, t3, 0x7632);
        uint32_t* d = reinterpret_cast<uint32_t*>(dst + (int64_t)(4 * j) * N) + i;
        d[0] = o0;
        d[N / 4] = o1;
        d[2 * (N / 4)] = o2;
        d[3 * (N / 4)] = o3;
    }
    if (t == 0) swT[((int64_t)e * KB + kb) * NB + nb] = sw[((int64_t)e * NB + nb) * KB + kb];
}

}  // namespace

extern "C" fg8_status fg8_transpose_blockq(const uint8_t* wq, const float* sw, int E, int N,
                                           int K, uint8_t* wqT, float* swT,
                                           fg8_stream_t stream) {
    if (!wq || !sw || !wqT || !swT) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (N / 128 > 65535 || E > 65535) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(wq) || !fg8h::aligned16(wqT)) return FG8_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sw) & 3) || (reinterpret_cast<uintptr_t>(swT) & 3))
        return FG8_ERR_INVALID_ARG;
    dim3 grid(K / 128, N / 128, E);
    transpose_blocks<<<grid, kThreads, 0, (cudaStream_t)stream>>>(wq, sw, N, K, wqT, swT);
    return fg8h::launch_status();
}
