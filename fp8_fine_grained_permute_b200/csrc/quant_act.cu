// quant_act.cu -- 1x128 activation quantization fused with the token-to-expert
// permute, for all experts in one launch (Kanana-2 deep dive, devday.kr, FP8
// paragraph: a MoE quantization kernel instead of one launch per expert;
// DeepSeek-V3 summary sec. 2.1: top-K routing without token dropping, so the
// permuted activation has exactly T*k rows; sec. 2.2: 1x128 tiles).
//
// Three kernels:
//  * route_quant   (permuting mode) -- one cooperative launch, three phases:
//      A  each CTA histograms the expert ids of its token chunk;
//      B  per expert, an exclusive scan of the chunk histograms (one warp per
//         expert) gives every chunk its first row inside each expert;
//      C  each CTA turns the expert totals into expert offsets, ranks its
//         (token, slot) pairs stably with warp match-any, writes the index
//         maps, then quantizes each of its token rows ONCE and stores the
//         codes to all k destination rows.
//    Phases are separated by grid-wide barriers with bounded waits.
//  * quant_rows    (rows already in expert order): the phase-C row loop only.
//  * colwise_tiles (weight-gradient operands): 128 tokens x 128 columns per
//    CTA, amax per column over the tile's tokens, codes written transposed so
//    that the token axis is contiguous.
#include <atomic>

#include "fg8_common.cuh"

namespace {

constexpr int kThreads = 512;            // route_quant / quant_rows
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 2048;               // experts supported by route_quant / colwise
constexpr int kMaxGrid = 1024;            // CTAs of route_quant (sizes the workspace)
constexpr unsigned kFull = 0xFFFFFFFFu;

// --------------------------------------------------------------------------
// shared helpers
// --------------------------------------------------------------------------

// Grid-wide barrier on a zero-initialised counter; `target` = CTAs * phase.
// Returns false (and records FG8_ERR_TIMEOUT) if the wait runs out.
__device__ bool grid_barrier(uint32_t* counter, uint32_t target, int32_t* status) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1u);
        const uint64_t t0 = fg8::globaltimer_ns();
        int ok = 1;
        while (fg8::ld_acquire_gpu(counter) < target) {
            if (fg8::globaltimer_ns() - t0 > fg8::kWaitLimitNs) {
                ok = 0;
                fg8::set_status(status, FG8_ERR_TIMEOUT);
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// Quantize one token row (K bf16, K % 128 == 0) in 1x128 tiles and store the
// codes into the `nd` rows held by lanes 0..nd-1 of `my_row` (negative rows
// are skipped).  The warp walks the row in 256-element segments: lane l holds
// elements 8l..8l+7, lanes 0-15 form one tile and lanes 16-31 the next.
__device__ __forceinline__ void quant_row(const uint16_t* __restrict__ src, int64_t K,
                                          int my_row, int nd, uint8_t* __restrict__ xq,
                                          float* __restrict__ sa, int64_t R, int lane) {
    const int nseg = (int)((K + 255) / 256);
    for (int s0 = 0; s0 < nseg; s0 += 4) {
        uint4 v[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t off = (int64_t)(s0 + u) * 256 + 8 * lane;
            ok[u] = (s0 + u < nseg) && (off < K);
            v[u] = ok[u] ? fg8::ld_stream16(src + off) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (s0 + u >= nseg) break;                 // warp-uniform
            float m = fg8::amax8(v[u]);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
            const float s = fg8::tile_scale(m);
            const fg8::QScale q = fg8::make_qscale(s);
            const uint2 c = fg8::quant8(v[u], q);
            const int64_t off = (int64_t)(s0 + u) * 256 + 8 * lane;
            const int64_t kb = (int64_t)(s0 + u) * 2 + (lane >> 4);
            for (int j = 0; j < nd; ++j) {
                const int r = __shfl_sync(kFull, my_row, j);
                if (ok[u] && r >= 0) {
                    *reinterpret_cast<uint2*>(xq + (int64_t)r * K + off) = c;
                    if ((lane & 15) == 0) sa[kb * R + r] = s;
                }
            }
        }
    }
}

// --------------------------------------------------------------------------
// permuting mode
// --------------------------------------------------------------------------

struct RouteArgs {
    const uint16_t* x;
    int64_t T, K;
    const int32_t* ids;
    int k, E;
    uint8_t* xq;
    float* sa;
    int32_t* row_token;
    int32_t* token_row;
    int32_t* offsets_out;
    uint32_t* bar;          // workspace: barrier counter
    int32_t* totals;        // workspace: [E]
    int32_t* chunk_counts;  // workspace: [gridDim.x][E]
    int32_t* status;
};

__global__ void __launch_bounds__(kThreads) route_quant(RouteArgs a) {
    __shared__ int32_t s_cnt[kMaxE];
    __shared__ int32_t s_off[kMaxE + 1];
    __shared__ int32_t s_warp[33];

    const int G = gridDim.x, c = blockIdx.x, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const int E = a.E, k = a.k;
    const int64_t t_begin = (int64_t)c * a.T / G, t_end = (int64_t)(c + 1) * a.T / G;
    const int64_t p_begin = t_begin * k, p_end = t_end * k;
    const int64_t R = a.T * k;

    // ---- phase A: chunk histogram
    for (int e = t; e < E; e += kThreads) s_cnt[e] = 0;
    __syncthreads();
    for (int64_t p = p_begin + t; p < p_end; p += kThreads) {
        const int32_t e = a.ids[p];
        if (e >= 0 && e < E)
            atomicAdd(&s_cnt[e], 1);
        else
            fg8::set_status(a.status, FG8_ERR_BAD_EXPERT_ID);
    }
    __syncthreads();
    for (int e = t; e < E; e += kThreads) a.chunk_counts[(int64_t)c * E + e] = s_cnt[e];
    if (!grid_barrier(a.bar, (uint32_t)G, a.status)) return;

    // ---- phase B: per expert, exclusive scan over chunks (one warp each)
    for (int e = c * kWarps + warp; e < E; e += G * kWarps) {
        int32_t carry = 0;
        for (int c0 = 0; c0 < G; c0 += 32) {
            const int cc = c0 + lane;
            const int32_t v = cc < G ? a.chunk_counts[(int64_t)cc * E + e] : 0;
            int32_t incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            if (cc < G) a.chunk_counts[(int64_t)cc * E + e] = carry + incl - v;
            carry += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) a.totals[e] = carry;
    }
    if (!grid_barrier(a.bar, 2u * (uint32_t)G, a.status)) return;

    // ---- phase C: offsets, stable ranks, index maps
    for (int e = t; e < E; e += kThreads) s_cnt[e] = a.totals[e];
    __syncthreads();
    fg8::block_exclusive_scan(s_cnt, s_off, E, s_warp);
    if (c == 0)
        for (int e = t; e <= E; e += kThreads) a.offsets_out[e] = s_off[e];
    // s_cnt becomes this chunk's next free row per expert
    for (int e = t; e < E; e += kThreads) s_cnt[e] = s_off[e] + a.chunk_counts[(int64_t)c * E + e];
    __syncthreads();
    if (warp == 0) {
        const unsigned lt = (1u << lane) - 1u;
        for (int64_t p0 = p_begin; p0 < p_end; p0 += 32) {
            const int64_t p = p0 + lane;
            const bool valid = p < p_end;
            const int32_t e = valid ? a.ids[p] : -1;
            const bool good = valid && e >= 0 && e < E;
            const int key = good ? e : (0x40000000 + lane);
            const unsigned m = __match_any_sync(kFull, key);
            const int32_t base = good ? s_cnt[e] : 0;
            const int32_t row = base + __popc(m & lt);
            __syncwarp();
            if (good && (__ffs(m) - 1) == lane) s_cnt[e] = base + __popc(m);
            __syncwarp();
            if (valid) {
                a.token_row[p] = good ? row : -1;
                if (good) a.row_token[row] = (int32_t)(p / k);
            }
        }
    }
    __syncthreads();

    // ---- phase C: quantize each token row once, store to its k rows
    for (int64_t tok = t_begin + warp; tok < t_end; tok += kWarps) {
        const int my_row = lane < k ? a.token_row[tok * k + lane] : -1;
        quant_row(a.x + tok * a.K, a.K, my_row, k, a.xq, a.sa, R, lane);
    }
}

// --------------------------------------------------------------------------
// identity mode
// --------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads)
quant_rows(const uint16_t* __restrict__ x, int64_t R, int64_t K, uint8_t* __restrict__ xq,
           float* __restrict__ sa) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t r = gw; r < R; r += nwarps)
        quant_row(x + r * K, K, lane == 0 ? (int)r : -1, 1, xq, sa, R, lane);
}

// --------------------------------------------------------------------------
// column-wise (token-axis) mode
// --------------------------------------------------------------------------

constexpr int kColThreads = 256;
constexpr int kXsStride = 130;   // bf16 per shared row (128 + 2): conflict-free column reads
constexpr int kTsStride = 144;   // bytes per staged code row (128 + 16), rows 16-byte aligned
// shared-memory map of colwise_tiles (byte offsets; ts rows are read as 16-byte vectors)
constexpr size_t kOffTs = 0;
constexpr size_t kOffXs = kOffTs + 128 * kTsStride;                        // 18432
constexpr size_t kOffScale = kOffXs + sizeof(uint16_t) * 128 * kXsStride;  // 51712
constexpr size_t kOffNtile = kOffScale + sizeof(float) * 128;
constexpr size_t kOffPref = kOffNtile + sizeof(int32_t) * kMaxE;
constexpr size_t kOffWarp = kOffPref + sizeof(int32_t) * (kMaxE + 4);
constexpr size_t kColSmem = kOffWarp + sizeof(int32_t) * 36;
static_assert(kOffTs % 16 == 0 && kTsStride % 16 == 0, "ts rows are read as 16-byte vectors");
static_assert(kOffXs % 4 == 0 && (kXsStride * 2) % 4 == 0, "xs rows are written as words");
static_assert(kOffScale % 4 == 0 && kOffNtile % 4 == 0 && kOffWarp % 4 == 0, "word arrays");

struct ColArgs {
    const uint16_t* x;
    int64_t T_src;          // rows of x
    int64_t R;              // logical rows
    int64_t C;
    const int32_t* row_map;
    const int32_t* offsets;
    int E;
    int64_t P;
    uint8_t* xqT;
    float* saT;
    int32_t* padoff_out;
};

__global__ void __launch_bounds__(kColThreads) colwise_tiles(ColArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* ts = smem + kOffTs;                                       // [128][kTsStride] codes
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + kOffXs);        // [128][kXsStride] bf16
    float* s_scale = reinterpret_cast<float*>(smem + kOffScale);      // [128]
    int32_t* s_ntile = reinterpret_cast<int32_t*>(smem + kOffNtile);  // [kMaxE]
    int32_t* s_pref = reinterpret_cast<int32_t*>(smem + kOffPref);    // [kMaxE + 1]
    int32_t* s_warp = reinterpret_cast<int32_t*>(smem + kOffWarp);    // [33]

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int E = a.E;

    for (int e = t; e < E; e += kColThreads) {
        const int32_t Te = max(0, a.offsets[e + 1] - a.offsets[e]);
        s_ntile[e] = (Te + 127) / 128;
    }
    __syncthreads();
    fg8::block_exclusive_scan(s_ntile, s_pref, E, s_warp);
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int e = t; e <= E; e += kColThreads) a.padoff_out[e] = 128 * s_pref[e];

    const int tile = blockIdx.x;
    if (tile >= s_pref[E]) return;   // block-uniform
    int lo = 0, hi = E;              // largest e with s_pref[e] <= tile
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pref[mid] <= tile) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int tb = tile - s_pref[e];
    const int32_t Te = a.offsets[e + 1] - a.offsets[e];
    const int n_in = min(128, Te - 128 * tb);
    const int64_t row0 = (int64_t)a.offsets[e] + 128 * tb;
    const int64_t col0 = (int64_t)blockIdx.y * 128;

    // load 128 rows x 128 columns (bf16) into shared memory, zeros past n_in
    {
        const int ch = t & 15, rr = t >> 4;
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int row = rr + 16 * i;
            v[i] = make_uint4(0u, 0u, 0u, 0u);
            const int64_t lr = row0 + row;
            if (row < n_in && lr < a.R) {
                const int64_t sr = a.row_map ? (int64_t)a.row_map[lr] : lr;
                if (sr >= 0 && sr < a.T_src) v[i] = fg8::ld_stream16(a.x + sr * a.C + col0 + ch * 8);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t* d = reinterpret_cast<uint32_t*>(xs + (rr + 16 * i) * kXsStride + ch * 8);
            d[0] = v[i].x; d[1] = v[i].y; d[2] = v[i].z; d[3] = v[i].w;
        }
    }
    __syncthreads();

    // per-column amax over the tile's rows (padding rows are zero)
    for (int cc = warp; cc < 128; cc += kColThreads / 32) {
        float m = 0.0f;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint16_t b = xs[(lane + 32 * g) * kXsStride + cc];
            m = fmaxf(m, fabsf(__uint_as_float((uint32_t)b << 16)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        if (lane == 0) s_scale[cc] = fg8::tile_scale(m);
    }
    __syncthreads();

    // quantize into the transposed staging tile: ts[column][token]
    for (int cc = warp; cc < 128; cc += kColThreads / 32) {
        const fg8::QScale q = fg8::make_qscale(s_scale[cc]);
#pragma unroll
        for (int g = 0; g < 4; g += 2) {
            const int row = lane + 32 * g;   // and row + 32
            const float x0 = __uint_as_float((uint32_t)xs[row * kXsStride + cc] << 16);
            const float x1 = __uint_as_float((uint32_t)xs[(row + 32) * kXsStride + cc] << 16);
            const uint32_t c = fg8::quant_pair(x0, x1, q);
            ts[cc * kTsStride + row] = (uint8_t)(c & 0xFFu);
            ts[cc * kTsStride + row + 32] = (uint8_t)(c >> 8);
        }
    }
    __syncthreads();

    const int64_t pcol = (int64_t)128 * s_pref[e] + 128 * tb;   // padded token column
    if (pcol + 128 > a.P) return;   // offsets inconsistent with R: never write past the buffers
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = t + kColThreads * i;
        const int cc = idx >> 3, ch = idx & 7;
        const uint4 v = *reinterpret_cast<const uint4*>(ts + cc * kTsStride + ch * 16);
        *reinterpret_cast<uint4*>(a.xqT + (col0 + cc) * a.P + pcol + ch * 16) = v;
    }
    if (t < 128) a.saT[(pcol / 128) * a.C + col0 + t] = s_scale[t];
}

size_t ws_layout(int64_t E, size_t* off_totals, size_t* off_chunks) {
    const size_t bar = 256;                                       // barrier counter(s)
    const size_t totals = ((size_t)E * 4 + 255) / 256 * 256;
    *off_totals = bar;
    *off_chunks = bar + totals;
    return bar + totals + (size_t)kMaxGrid * (size_t)E * 4;
}

}  // namespace

extern "C" size_t fg8_quantize_act_workspace(int64_t T, int k, int E) {
    (void)T;
    (void)k;
    if (E < 1) return 0;
    size_t a, b;
    return ws_layout(E, &a, &b);
}

extern "C" int64_t fg8_colwise_capacity(int64_t R, int E) {
    return (R + 127 * (int64_t)E + 127) / 128 * 128;
}

extern "C" fg8_status fg8_quantize_act(const uint16_t* x, int64_t T, int64_t K,
                                       const int32_t* topk_ids, int k, int E,
                                       const int32_t* offsets_in, int layout,
                                       uint8_t* xq, float* sa,
                                       int32_t* row_token, int32_t* token_row,
                                       int32_t* offsets_out, uint8_t* xqT, float* saT,
                                       void* workspace, size_t ws_bytes,
                                       int32_t* dev_status, fg8_stream_t stream) {
    cudaStream_t st = (cudaStream_t)stream;
    if (T < 0 || K < 128 || K % 128 || k < 1) return FG8_ERR_INVALID_ARG;
    if (x == nullptr && T > 0) return FG8_ERR_INVALID_ARG;
    if (x && !fg8h::aligned16(x)) return FG8_ERR_INVALID_ARG;

    // no tokens: the permuting mode still reports empty experts (the id buffer of
    // an empty batch may be NULL); the other modes have nothing to do
    if (layout == FG8_ROWWISE && T == 0 && offsets_out != nullptr) {
        if (E < 1) return FG8_ERR_INVALID_ARG;
        return cudaMemsetAsync(offsets_out, 0, sizeof(int32_t) * ((size_t)E + 1), st) == cudaSuccess
                   ? FG8_OK : FG8_ERR_CUDA;
    }

    if (layout == FG8_ROWWISE && topk_ids == nullptr) {
        if (k != 1) return FG8_ERR_INVALID_ARG;
        if (T == 0) return FG8_OK;
        if (!xq || !sa) return FG8_ERR_INVALID_ARG;
        if (!fg8h::aligned16(xq) || (reinterpret_cast<uintptr_t>(sa) & 3)) return FG8_ERR_INVALID_ARG;
        const int64_t warps_needed = T;
        int64_t blocks = (warps_needed + kWarps - 1) / kWarps;
        const int64_t cap = (int64_t)fg8h::num_sms() * 4;
        if (blocks > cap) blocks = cap;
        quant_rows<<<(unsigned)blocks, kThreads, 0, st>>>(x, T, K, xq, sa);
        return fg8h::launch_status();
    }

    if (layout == FG8_ROWWISE) {
        if (E < 1 || k > 32) return E < 1 ? FG8_ERR_INVALID_ARG : FG8_ERR_UNSUPPORTED;
        if (E > kMaxE) return FG8_ERR_UNSUPPORTED;
        if (!xq || !sa || !row_token || !token_row || !offsets_out || !workspace)
            return FG8_ERR_INVALID_ARG;
        if (!fg8h::aligned16(xq) || !fg8h::aligned16(workspace)) return FG8_ERR_INVALID_ARG;
        if (T * k > (int64_t)INT32_MAX) return FG8_ERR_UNSUPPORTED;
        size_t off_tot, off_chk;
        const size_t need = ws_layout(E, &off_tot, &off_chk);
        if (ws_bytes < need) return FG8_ERR_INVALID_ARG;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_quant, kThreads, 0) !=
                cudaSuccess || per_sm < 1)
            return FG8_ERR_CUDA;
        int64_t G = (int64_t)per_sm * fg8h::num_sms();
        if (G > kMaxGrid) G = kMaxGrid;
        if (G > (T + 1) / 2) G = (T + 1) / 2;
        if (G < 1) G = 1;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return FG8_ERR_CUDA;
        RouteArgs a;
        a.x = x; a.T = T; a.K = K; a.ids = topk_ids; a.k = k; a.E = E;
        a.xq = xq; a.sa = sa; a.row_token = row_token; a.token_row = token_row;
        a.offsets_out = offsets_out;
        a.bar = reinterpret_cast<uint32_t*>(ws);
        a.totals = reinterpret_cast<int32_t*>(ws + off_tot);
        a.chunk_counts = reinterpret_cast<int32_t*>(ws + off_chk);
        a.status = dev_status;
        void* args[] = {&a};
        if (cudaLaunchCooperativeKernel((const void*)route_quant, dim3((unsigned)G), dim3(kThreads),
                                        args, 0, st) != cudaSuccess)
            return FG8_ERR_CUDA;
        return fg8h::launch_status();
    }

    if (layout == FG8_COLWISE) {
        if (E < 1 || E > kMaxE) return E > kMaxE ? FG8_ERR_UNSUPPORTED : FG8_ERR_INVALID_ARG;
        if (!offsets_in || !xqT || !saT || !offsets_out) return FG8_ERR_INVALID_ARG;
        if (row_token == nullptr && k != 1) return FG8_ERR_INVALID_ARG;
        if (!fg8h::aligned16(xqT) || !fg8h::aligned16(saT)) return FG8_ERR_INVALID_ARG;
        if (K / 128 > 65535) return FG8_ERR_UNSUPPORTED;
        const int64_t R = T * k;
        const int64_t P = fg8_colwise_capacity(R, E);
        const int64_t max_tiles = R / 128 + E;
        if (max_tiles > INT32_MAX) return FG8_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(colwise_tiles, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kColSmem) != cudaSuccess)
            return FG8_ERR_CUDA;
        ColArgs a;
        a.x = x; a.T_src = T; a.R = R; a.C = K; a.row_map = row_token; a.offsets = offsets_in; a.E = E; a.P = P;
        a.xqT = xqT; a.saT = saT; a.padoff_out = offsets_out;
        dim3 grid((unsigned)max_tiles, (unsigned)(K / 128));
        colwise_tiles<<<grid, kColThreads, kColSmem, st>>>(a);
        return fg8h::launch_status();
    }
    return FG8_ERR_INVALID_ARG;
}

// --------------------------------------------------------------------------
// permuting mode without a caller-provided workspace
// --------------------------------------------------------------------------
//
// Some callers have no way to allocate device memory: a plugin interface of a
// host framework that owns every device allocation and hands a kernel only its
// inputs and outputs, or a latency-critical path that must never enter the
// allocator.  For them the permuting mode can use a scratch area that lives in
// the library itself: a file-scope __device__ array, which every GPU that
// loads libfg8 holds until the process exits.  It is sized for up to
// kNoAllocMaxExperts experts; larger E is rejected.
//
// Host code cannot use the array's name as a device address (it is a host-side
// stand-in), so on the first call on each device, with that device current,
// the entry point asks the runtime for the array's device address and caches
// it.  That first call should therefore come before any stream capture.

namespace {

constexpr int kNoAllocMaxExperts = 256;
constexpr size_t kNoAllocScratchBytes =
    256 + 4 * (size_t)kNoAllocMaxExperts + (size_t)kMaxGrid * kNoAllocMaxExperts * 4;  // ~1 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_noalloc_addr[kMaxDevices];

}  // namespace

extern "C" fg8_status fg8_quantize_act_noalloc(const uint16_t* x, int64_t T, int64_t K,
                                               const int32_t* topk_ids, int k, int E,
                                               uint8_t* xq, float* sa, int32_t* row_token,
                                               int32_t* token_row, int32_t* offsets_out,
                                               int32_t* dev_status, fg8_stream_t stream) {
    if (E < 1) return FG8_ERR_INVALID_ARG;
    if (E > kNoAllocMaxExperts) return FG8_ERR_UNSUPPORTED;
    size_t off_tot, off_chk;
    const size_t need = ws_layout(E, &off_tot, &off_chk);
    if (need > kNoAllocScratchBytes) return FG8_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FG8_ERR_CUDA;
    void* scratch = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (scratch == nullptr) {
        if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr)
            return FG8_ERR_CUDA;
        g_noalloc_addr[dev].store(scratch, std::memory_order_release);
    }
    // the permuting entry point clears the barrier word on every call; the
    // per-chunk counts and totals are fully written before they are read
    return fg8_quantize_act(x, T, K, topk_ids, k, E, nullptr, FG8_ROWWISE, xq, sa, row_token,
                            token_row, offsets_out, nullptr, nullptr, scratch,
                            kNoAllocScratchBytes, dev_status, stream);
}
