// ep.cu -- data plane of the expert-parallel exchange of FP8 rows.
//
// With the experts spread over W ranks (rank r owns the E_loc = E / W
// experts [r E_loc, (r + 1) E_loc)), every routed row has to reach the rank
// that owns its expert, and the expert output has to come back for the
// combine (the all-to-all dispatch and combine of expert parallelism, with
// the FP8 codes and their 1x128 scales crossing the links instead of bf16:
// DeepSeek-V3 summary sec. 2.2 on the NVLink / InfiniBand cluster and FP8
// communication; the Pangu/Ascend article's expert-parallel all-to-all).
//
// The permuting quantizer has already grouped the rows by expert in
// ascending order, so each destination's rows are one contiguous range of
// xq and go out as they are.  What this file adds:
//   ep_pack_scales   sa [K/128][R] -> one scale row per routed row [R][K/128],
//                    so a row's scales travel next to its codes;
//   ep_unpack        on the receiver, the W incoming segments (each grouped
//                    by local expert) -> local expert order, expert-major and
//                    then by source rank: codes [R_recv][K], scales in the
//                    GEMM's [K/128][R_recv] layout, local expert offsets, and
//                    the received-row -> local-row map;
//   gather_rows      out[i] = in[map[i]]: the combine sends each expert
//                    output row back in the order it was received.
// The exchange itself (counts, then codes and scales, then outputs) is NCCL
// all-to-all driven by the host; no TMA multicast load reads peer memory.
#include "fg8_common.cuh"

namespace {

constexpr int kMaxSeg = 2048;   // W * E_loc segments handled by ep_unpack (8 per thread)

// ---------------------------------------------------------------------------
// scale rows: [KB][R] -> [R][KB], 32 x 32 tiles through shared memory
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ep_pack_scales(const float* __restrict__ sa, int64_t R, int KB,
                                                      float* __restrict__ sa_rows) {
    __shared__ float tile[32][33];
    const int64_t r0 = (int64_t)blockIdx.x * 32;
    const int kb0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        const int kb = kb0 + ty + i;
        const int64_t r = r0 + tx;
        if (kb < KB && r < R) tile[ty + i][tx] = sa[(int64_t)kb * R + r];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        const int64_t r = r0 + ty + i;
        const int kb = kb0 + tx;
        if (kb < KB && r < R) sa_rows[r * KB + kb] = tile[tx][ty + i];
    }
}

// ---------------------------------------------------------------------------
// receiver side: segments (source s, local expert e) -> local expert order
// ---------------------------------------------------------------------------
struct UnpackArgs {
    const uint8_t* recv_xq;       // [R_recv][K]
    const float* recv_sa;         // [R_recv][KB]
    const int32_t* counts;        // [W][E_loc]: rows source s sent for local expert e
    int W, E_loc;
    int64_t R_recv;
    int64_t K;
    uint8_t* xq;                  // [R_recv][K], local expert order
    float* sa;                    // [KB][R_recv]
    int32_t* offsets;             // [E_loc + 1]
    int32_t* recv_to_local;       // [R_recv]
    int32_t* status;
};

// Every CTA rebuilds the (small) segment tables in shared memory with two
// block scans -- the received order is source-major, the local order
// expert-major -- then copies rows grid-stride, one warp per row (16-byte
// vectors for the codes).
__global__ void __launch_bounds__(256) ep_unpack(UnpackArgs a) {
    __shared__ int32_t s_cnt[kMaxSeg];
    __shared__ int32_t s_src[kMaxSeg + 1];   // first received row of segment s * E_loc + e
    __shared__ int32_t s_dst[kMaxSeg + 1];   // first local row of segment e * W + s
    __shared__ int32_t s_warp[33];
    const int W = a.W, EL = a.E_loc, nseg = W * EL;
    const int t = threadIdx.x, lane = t & 31;
    for (int i = t; i < nseg; i += blockDim.x) s_cnt[i] = max(0, a.counts[i]);
    __syncthreads();
    fg8::block_exclusive_scan(s_cnt, s_src, nseg, s_warp);
    // expert-major copy of the counts, scanned in place
    for (int i = t; i < nseg; i += blockDim.x) {
        const int e = i / W, s = i - e * W;
        s_dst[i] = s_cnt[s * EL + e];
    }
    __syncthreads();
    fg8::block_exclusive_scan(s_dst, s_dst, nseg, s_warp);
    if (s_src[nseg] != a.R_recv) {   // counts disagree with the buffers: nothing written
        if (blockIdx.x == 0 && t == 0) fg8::set_status(a.status, FG8_ERR_INVALID_ARG);
        return;
    }
    if (blockIdx.x == 0) {
        for (int e = t; e < EL; e += blockDim.x) a.offsets[e] = s_dst[e * W];
        if (t == 0) a.offsets[EL] = s_dst[nseg];
    }
    const int KB = (int)(a.K / 128);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    int seg = 0;
    for (int64_t j = (int64_t)blockIdx.x * (blockDim.x >> 5) + (t >> 5); j < a.R_recv; j += nwarps) {
        // segment (source-major index) holding received row j: the last one
        // starting at or before j (rows only increase, so the previous one is
        // tried first)
        if (s_src[seg] > j || s_src[seg + 1] <= j) {
            int lo = 0, hi = nseg;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_src[mid] <= j) lo = mid; else hi = mid;
            }
            seg = lo;
        }
        const int s = seg / EL, e = seg - s * EL;
        const int64_t dst = (int64_t)s_dst[e * W + s] + (j - s_src[seg]);
        const uint4* src = reinterpret_cast<const uint4*>(a.recv_xq + j * a.K);
        uint4* out = reinterpret_cast<uint4*>(a.xq + dst * a.K);
        for (int64_t v = lane; v < a.K / 16; v += 32) out[v] = fg8::ld_stream16(src + v);
        for (int kb = lane; kb < KB; kb += 32) a.sa[(int64_t)kb * a.R_recv + dst] = a.recv_sa[j * KB + kb];
        if (lane == 0) a.recv_to_local[j] = (int32_t)dst;
    }
}

// ---------------------------------------------------------------------------
// out[i] = in[map[i]] for rows of `row_bytes` (a multiple of 16)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows(const uint8_t* __restrict__ in, int64_t n_in,
                                                   int64_t row_bytes, const int32_t* __restrict__ map,
                                                   int64_t n, uint8_t* __restrict__ out,
                                                   int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n; i += nwarps) {
        const int64_t m = map[i];
        if (m < 0 || m >= n_in) {   // not a row: report, leave the output row alone
            if (lane == 0) fg8::set_status(status, FG8_ERR_INVALID_ARG);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(in + m * row_bytes);
        uint4* dst = reinterpret_cast<uint4*>(out + i * row_bytes);
        for (int64_t v = lane; v < row_bytes / 16; v += 32) dst[v] = fg8::ld_stream16(src + v);
    }
}

int64_t rows_grid(int64_t rows) {
    const int64_t cap = 8 * (int64_t)fg8h::num_sms();
    int64_t g = (rows + 7) / 8;   // 8 warps per CTA, one row each
    if (g > cap) g = cap;
    return g < 1 ? 1 : g;
}

}  // namespace

extern "C" fg8_status fg8_ep_pack_scales(const float* sa, int64_t R, int64_t K, float* sa_rows,
                                         fg8_stream_t stream) {
    if (R < 0 || K < 128 || K % 128) return FG8_ERR_INVALID_ARG;
    if (R == 0) return FG8_OK;
    if (!sa || !sa_rows || (reinterpret_cast<uintptr_t>(sa) & 3) ||
        (reinterpret_cast<uintptr_t>(sa_rows) & 3))
        return FG8_ERR_INVALID_ARG;
    const int KB = (int)(K / 128);
    if ((R + 31) / 32 > INT32_MAX || (KB + 31) / 32 > 65535) return FG8_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((R + 31) / 32), (unsigned)((KB + 31) / 32));
    ep_pack_scales<<<grid, 256, 0, (cudaStream_t)stream>>>(sa, R, KB, sa_rows);
    return fg8h::launch_status();
}

extern "C" fg8_status fg8_ep_unpack(const uint8_t* recv_xq, const float* recv_sa,
                                    const int32_t* counts, int W, int E_loc, int64_t R_recv,
                                    int64_t K, uint8_t* xq, float* sa, int32_t* offsets,
                                    int32_t* recv_to_local, int32_t* dev_status,
                                    fg8_stream_t stream) {
    if (W < 1 || E_loc < 1 || (int64_t)W * E_loc > kMaxSeg || R_recv < 0 ||
        K < 128 || K % 128)
        return FG8_ERR_INVALID_ARG;
    if (!counts || !offsets) return FG8_ERR_INVALID_ARG;
    if (R_recv > 0 && (!recv_xq || !recv_sa || !xq || !sa || !recv_to_local))
        return FG8_ERR_INVALID_ARG;
    if (R_recv > INT32_MAX) return FG8_ERR_UNSUPPORTED;
    if ((R_recv > 0 && (!fg8h::aligned16(recv_xq) || !fg8h::aligned16(xq))) ||
        (reinterpret_cast<uintptr_t>(recv_sa) & 3) || (reinterpret_cast<uintptr_t>(sa) & 3) ||
        (reinterpret_cast<uintptr_t>(counts) & 3))
        return FG8_ERR_INVALID_ARG;
    UnpackArgs a;
    a.recv_xq = recv_xq; a.recv_sa = recv_sa; a.counts = counts; a.W = W; a.E_loc = E_loc;
    a.R_recv = R_recv; a.K = K; a.xq = xq; a.sa = sa; a.offsets = offsets;
    a.recv_to_local = recv_to_local; a.status = dev_status;
    ep_unpack<<<(unsigned)rows_grid(R_recv), 256, 0, (cudaStream_t)stream>>>(a);
    return fg8h::launch_status();
}

extern "C" fg8_status fg8_gather_rows(const void* in, int64_t n_in, int64_t row_bytes,
                                      const int32_t* map, int64_t n, void* out,
                                      int32_t* dev_status, fg8_stream_t stream) {
    if (n < 0 || n_in < 0 || row_bytes < 16 || row_bytes % 16) return FG8_ERR_INVALID_ARG;
    if (n == 0) return FG8_OK;
    if (!in || !map || !out || !fg8h::aligned16(in) || !fg8h::aligned16(out) ||
        (reinterpret_cast<uintptr_t>(map) & 3))
        return FG8_ERR_INVALID_ARG;
    gather_rows<<<(unsigned)rows_grid(n), 256, 0, (cudaStream_t)stream>>>(
        static_cast<const uint8_t*>(in), n_in, row_bytes, map, n, static_cast<uint8_t*>(out),
        dev_status);
    return fg8h::launch_status();
}
