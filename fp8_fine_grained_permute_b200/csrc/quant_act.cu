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
//  * quant_rows    (rows already in expert order): 128 x 128 boxes staged in
//    shared memory by one TMA load each, eight lanes per row tile.
//  * colwise_tiles (weight-gradient operands): one 128-token tile x a quarter
//    of the columns per CTA, 128 columns at a time through a two-stage
//    cp.async pipeline; amax per column over the tile's tokens, codes written
//    transposed so that the token axis is contiguous (thread = 2 columns x 32
//    tokens).
//  quant_rows and colwise_tiles convert with the branch-free fast path and
//  redo the groups whose bracket check failed after their main loop (per
//  128-column block for colwise_tiles), shared out over the warp.
#include <cuda.h>

#include <mutex>

#include "fg8_common.cuh"
#include "fg8_route.cuh"
#include "fg8_tma.cuh"

namespace {

constexpr int kThreads = 512;            // route_quant
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 2048;               // experts supported by route_quant / colwise
constexpr int kMaxGrid = 1024;            // CTAs of route_quant (sizes the workspace)
constexpr unsigned kFull = 0xFFFFFFFFu;

// --------------------------------------------------------------------------
// shared helpers
// --------------------------------------------------------------------------

// Quantize one token row (K bf16, K % 128 == 0) in 1x128 tiles and store the
// codes into the `nd` rows held by lanes 0..nd-1 of `my_row` (negative rows
// are skipped).  Eight lanes own one tile (16 values each: 16-byte chunks j and
// j + 8, so a warp's loads are whole 128-byte lines), a warp four tiles at a
// time, two such groups (eight tiles) in flight per iteration; the tile scale
// is computed once per 16 values.  Neighbouring lanes then swap one 8-byte
// half of their codes, so that each lane holds 16 consecutive codes (even
// lane j: chunks j, j + 1; odd lane j: chunks j + 7, j + 8) and writes every
// destination row with one aligned 16-byte store.
// Tiles [t_lo, t_hi) of the row are done (t_lo a multiple of 8).
__device__ __forceinline__ void quant_row(const uint16_t* __restrict__ src, int64_t K,
                                          int my_row, int nd, uint8_t* __restrict__ xq,
                                          float* __restrict__ sa, int64_t R, int lane,
                                          int t_lo, int t_hi) {
    const int ntile = t_hi;
    const int g = lane >> 3, j = lane & 7;
    for (int t0 = t_lo; t0 < ntile; t0 += 8) {
        uint4 v[2][2];
        bool ok[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int tile = t0 + 4 * u + g;
            ok[u] = tile < ntile;
            const uint16_t* p = src + (int64_t)tile * 128 + 8 * j;
            v[u][0] = ok[u] ? fg8::ld_stream16(p) : make_uint4(0u, 0u, 0u, 0u);
            v[u][1] = ok[u] ? fg8::ld_stream16(p + 64) : make_uint4(0u, 0u, 0u, 0u);
        }
        float m[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) m[u] = fmaxf(fg8::amax8(v[u][0]), fg8::amax8(v[u][1]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < 2; ++u) m[u] = fmaxf(m[u], __shfl_xor_sync(kFull, m[u], o));
        // fast-path codes of both groups first, one combined check
        float s[2];
        fg8::QScale q[2];
        uint2 c[2][2], h[2][2];
        bool fast = true;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            s[u] = fg8::tile_scale(m[u]);
            q[u] = fg8::make_qscale(s[u]);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                fg8::quant8_bracket(v[u][x], q[u], c[u][x], h[u][x]);
                fast &= !q[u].exact && fg8::bracket_agrees(c[u][x], h[u][x]);
            }
        }
        if (!fast) {
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int x = 0; x < 2; ++x)
                    if (q[u].exact || !fg8::bracket_agrees(c[u][x], h[u][x]))
                        c[u][x] = fg8::quant8_exact(v[u][x], q[u]);
        }
        const bool even = (j & 1) == 0;
        uint4 w16[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint2 give = even ? c[u][1] : c[u][0];
            uint2 got;
            got.x = __shfl_xor_sync(kFull, give.x, 1);
            got.y = __shfl_xor_sync(kFull, give.y, 1);
            w16[u] = even ? make_uint4(c[u][0].x, c[u][0].y, got.x, got.y)
                          : make_uint4(got.x, got.y, c[u][1].x, c[u][1].y);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int tile = t0 + 4 * u + g;
            const int64_t off = (int64_t)tile * 128 + 8 * j + (even ? 0 : 56);
            for (int d = 0; d < nd; ++d) {
                const int r = __shfl_sync(kFull, my_row, d);
                if (ok[u] && r >= 0) {
                    *reinterpret_cast<uint4*>(xq + (int64_t)r * K + off) = w16[u];
                    if (j == 0) sa[(int64_t)tile * R + r] = s[u];
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
    // fused routing (fg8_route_quantize_act): the ids are produced by the
    // kernel itself from router logits and the per-expert bias
    const float* logits;
    const float* bias;
    int32_t* ids_out;
    float* affinity;
};

// Shared memory of the permuting kernels.
struct RouteSmem {
    int32_t cnt[kMaxE];
    int32_t off[kMaxE + 1];
    int32_t warp[33];
};

// Phases B and C of the permuting kernels, after every CTA has written its
// chunk histogram to a.chunk_counts and passed the first grid barrier.
__device__ __forceinline__ void route_quant_scan_place_quantize(const RouteArgs& a, RouteSmem& sm) {
    const int G = gridDim.x, c = blockIdx.x, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const int E = a.E, k = a.k;
    const int64_t t_begin = (int64_t)c * a.T / G, t_end = (int64_t)(c + 1) * a.T / G;
    const int64_t p_begin = t_begin * k, p_end = t_end * k;
    const int64_t R = a.T * k;
    int32_t* s_cnt = sm.cnt;
    int32_t* s_off = sm.off;

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
    if (!fg8::grid_barrier(a.bar, 2u * (uint32_t)G, a.status)) return;

    // ---- phase C: offsets, stable ranks, index maps
    for (int e = t; e < E; e += kThreads) s_cnt[e] = a.totals[e];
    __syncthreads();
    fg8::block_exclusive_scan(s_cnt, s_off, E, sm.warp);
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

    // ---- phase C: quantize each token row once, store to its k rows.  The
    // work items are pieces of 8 tiles (1024 columns) of the chunk's token
    // rows, dealt to the warps in turn, so that every warp gets about the same
    // share however few tokens the chunk has.
    const int ntile = (int)(a.K / 128);
    const int pieces = (ntile + 7) / 8;
    const int64_t items = (t_end - t_begin) * pieces;
    for (int64_t it = warp; it < items; it += kWarps) {
        const int64_t tok = t_begin + it / pieces;
        const int pc = (int)(it % pieces);
        const int my_row = lane < k ? a.token_row[tok * k + lane] : -1;
        quant_row(a.x + tok * a.K, a.K, my_row, k, a.xq, a.sa, R, lane, 8 * pc, min(ntile, 8 * pc + 8));
    }
}

__global__ void __launch_bounds__(kThreads, 2) route_quant(RouteArgs a) {
    __shared__ RouteSmem sm;
    const int G = gridDim.x, c = blockIdx.x, t = threadIdx.x;
    const int E = a.E, k = a.k;
    const int64_t t_begin = (int64_t)c * a.T / G, t_end = (int64_t)(c + 1) * a.T / G;

    // ---- phase A: chunk histogram of the given ids
    for (int e = t; e < E; e += kThreads) sm.cnt[e] = 0;
    __syncthreads();
    for (int64_t p = t_begin * k + t; p < t_end * k; p += kThreads) {
        const int32_t e = a.ids[p];
        if (e >= 0 && e < E)
            atomicAdd(&sm.cnt[e], 1);
        else
            fg8::set_status(a.status, FG8_ERR_BAD_EXPERT_ID);
    }
    __syncthreads();
    for (int e = t; e < E; e += kThreads) a.chunk_counts[(int64_t)c * E + e] = sm.cnt[e];
    if (!fg8::grid_barrier(a.bar, (uint32_t)G, a.status)) return;
    route_quant_scan_place_quantize(a, sm);
}

// Routing fused in front of the permute: phase A routes this CTA's tokens
// (sigmoid affinity + bias, top-k, one warp per token, DeepSeek-V3 summary
// sec. 2.1), writes their ids and affinities and histograms the chosen
// experts in the same pass; phases B and C are those of route_quant (phase C
// reads back the ids this CTA has just written).  PER_LANE * 32 >= E.
template <int PER_LANE>
__global__ void __launch_bounds__(kThreads, PER_LANE >= 16 ? 1 : 2) route_topk_quant(RouteArgs a) {
    __shared__ RouteSmem sm;
    const int G = gridDim.x, c = blockIdx.x, t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const int E = a.E, k = a.k;
    const int64_t t_begin = (int64_t)c * a.T / G, t_end = (int64_t)(c + 1) * a.T / G;

    // ---- phase A: route the chunk's tokens, histogram the choices
    for (int e = t; e < E; e += kThreads) sm.cnt[e] = 0;
    float bl[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        bl[i] = e < E ? a.bias[e] : 0.f;
    }
    __syncthreads();
    for (int64_t tok = t_begin + warp; tok < t_end; tok += kWarps) {
        int32_t id;
        float sv;
        fg8::route_token<PER_LANE>(a.logits + tok * E, bl, E, k, lane, id, sv);
        if (lane < k) {
            a.ids_out[tok * k + lane] = id;
            a.affinity[tok * k + lane] = sv;
            atomicAdd(&sm.cnt[id], 1);
        }
    }
    __syncthreads();
    for (int e = t; e < E; e += kThreads) a.chunk_counts[(int64_t)c * E + e] = sm.cnt[e];
    if (!fg8::grid_barrier(a.bar, (uint32_t)G, a.status)) return;
    route_quant_scan_place_quantize(a, sm);
}

// --------------------------------------------------------------------------
// identity mode
// --------------------------------------------------------------------------

// One CTA per 128 rows x 128 columns: one 2-D TMA load stages the box (32 KB,
// rows past R read as zeros) in shared memory, five CTAs per SM keep the
// loads in flight.  Eight lanes own one row's 1x128 tile at a time (16 values
// each, chunks l and l + 8 so a warp's shared reads are conflict-free): amax
// by a 3-step shuffle, then the bracketed fast path; the tile's scale is
// computed once per 16 values (a half-warp per tile was 8% slower).
constexpr int kRowThreads = 256;
constexpr int kFixCap = 64;   // failed groups a warp redoes together
constexpr uint32_t kRowBoxBytes = 128 * 256;

__global__ void __launch_bounds__(kRowThreads, 5)
quant_rows(const __grid_constant__ CUtensorMap tmX, int64_t R, int64_t K, uint8_t* __restrict__ xq,
           float* __restrict__ sa, int32_t* status) {
    extern __shared__ __align__(128) uint8_t box[];   // [128 rows][256 bytes]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_abort;
    __shared__ float s_sc[kRowThreads / 32][16];               // each warp's 16 row scales
    __shared__ uint16_t s_fix[kRowThreads / 32][kFixCap];
    const int kb = blockIdx.x;
    const int64_t r0 = (int64_t)blockIdx.y * 128;
    const int t = threadIdx.x;
    const uint32_t bar = fg8::tma::smem_u32(&s_bar);
    if (t == 0) {
        s_abort = 0;
        fg8::tma::mbar_init(bar, 1);
        fg8::tma::fence_barrier_init();
        fg8::tma::mbar_arrive_expect_tx(bar, kRowBoxBytes);
        fg8::tma::tma_load_2d(&tmX, fg8::tma::smem_u32(box), bar, kb * 128, (int)r0);
    }
    __syncthreads();
    if (!fg8::tma::mbar_wait(bar, 0, &s_abort, status)) return;   // block-uniform in practice
    const int grp = t >> 3;        // 32 groups of 8 lanes: rows grp + 32 i
    const int l = t & 7;           // 16-byte chunks l and l + 8 of the row's tile
    // Groups whose fast path failed are only recorded here (bit 2 i + h) and
    // redone after the loop from the staged box, so the loop stays branch-free.
    uint32_t redo = 0;
    const int warp = t >> 5;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rr = grp + 32 * i;
        uint4 v[2];
        v[0] = *reinterpret_cast<const uint4*>(box + rr * 256 + l * 16);
        v[1] = *reinterpret_cast<const uint4*>(box + rr * 256 + 128 + l * 16);
        float m = fmaxf(fg8::amax8(v[0]), fg8::amax8(v[1]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        const float sc = fg8::tile_scale(m);
        if (l == 0) s_sc[warp][4 * i + (grp & 3)] = sc;
        const fg8::QScale q = fg8::make_qscale(sc);
        uint2 c[2], h[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            fg8::quant8_bracket(v[x], q, c[x], h[x]);
            redo |= (uint32_t)(q.exact || !fg8::bracket_agrees(c[x], h[x])) << (2 * i + x);
        }
        const int64_t r = r0 + rr;
        if (r < R) {
            uint8_t* d = xq + r * K + (int64_t)kb * 128 + l * 8;
            *reinterpret_cast<uint2*>(d) = c[0];
            *reinterpret_cast<uint2*>(d + 64) = c[1];
            if (l == 0) sa[(int64_t)kb * R + r] = sc;
        }
    }
    // the exact codes of those groups over the fast-path ones, shared out over
    // the warp (the fast-path stores were made before the warp barrier)
    auto redo_group = [&](int owner, int b) {
        const int to = 32 * warp + owner;
        const int og = to >> 3, ol = to & 7, i = b >> 1, x = b & 1;
        const int rr = og + 32 * i;
        const int64_t r = r0 + rr;
        const uint4 v = *reinterpret_cast<const uint4*>(box + rr * 256 + 128 * x + ol * 16);
        const uint2 c = fg8::quant8_redo(v, fg8::make_qscale(s_sc[warp][4 * i + (og & 3)]));
        if (r < R) *reinterpret_cast<uint2*>(xq + r * K + (int64_t)kb * 128 + ol * 8 + 64 * x) = c;
    };
    __syncwarp();   // the row scales
    if (!fg8::coop_redo(redo, s_fix[warp], kFixCap, redo_group)) {
        while (redo != 0u) {
            const int b = __ffs(redo) - 1;
            redo &= redo - 1u;
            redo_group(t & 31, b);
        }
    }
}

// --------------------------------------------------------------------------
// column-wise (token-axis) mode
// --------------------------------------------------------------------------

constexpr int kColThreads = 256;

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
    int32_t* status;
};

// One CTA per 128-token tile of one expert and per group of 128-column blocks
// (a quarter of the columns).  The tile's source rows (contiguous, or gathered
// through row_map) are found once; then, for each column block in turn, the
// 128 x 256-byte slice is brought into shared memory by cp.async (16 bytes a
// thread-copy, padding rows zero-filled), two stages deep, so the next block's
// data is in flight while this one is converted; one block barrier per column
// block.  Warp wp owns the column pairs 8 wp .. 8 wp + 7, lane 8 q + pl the 32
// tokens of quarter q of pair p = 8 wp + pl: it reads them as 32-bit words
// (rows are stored XOR-swizzled by quarter, so the warp's reads hit 32 banks),
// reduces its two column maxima in registers (16-bit SIMD max) and combines
// the quarters with two shuffles.  Codes are then formed per column on 8
// consecutive tokens at a time (bracketed fast path) and stored transposed:
// 32 contiguous bytes (a whole sector) of each column per thread.  (Measured
// against one CTA per 128 x 128 tile with the expert prefix recomputed by
// every CTA: 25% slower; against the quarters combined through shared
// memory with a second barrier: 4% slower.)
constexpr uint32_t kColTileBytes = 128 * 256;
constexpr int kColCtasPerSm = 3;
constexpr int kColFixCap = 64;   // failed groups a warp redoes together
// the warps' lists (from byte 0) and column-pair scales (from byte 2048) reuse s_pref
static_assert((kColThreads / 32) * kColFixCap * 2 <= 2048 &&
                  2048 + (kColThreads / 32) * 8 * 8 <= (kMaxE + 1) * 4,
              "column-wise redo lists fit the tile prefix array");
constexpr int kColGroups = 4;      // column groups per tile (grid.y)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__global__ void __launch_bounds__(kColThreads, kColCtasPerSm) colwise_tiles(ColArgs a) {
    extern __shared__ __align__(128) uint8_t s_tile[];   // [2][128 rows][256 bytes]
    // tiles per expert (prefix) while the CTA finds its tile; afterwards each
    // warp's list of failed groups and its 8 column-pair scales
    __shared__ __align__(16) int32_t s_pref[kMaxE + 1];
    __shared__ int32_t s_warp[33];
    __shared__ int32_t s_rows[128];

    const int t = threadIdx.x;
    const int E = a.E;
    for (int e = t; e < E; e += kColThreads) {
        const int32_t Te = max(0, a.offsets[e + 1] - a.offsets[e]);
        s_pref[e] = (Te + 127) / 128;
    }
    __syncthreads();
    fg8::block_exclusive_scan(s_pref, s_pref, E, s_warp);
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int e = t; e <= E; e += kColThreads) a.padoff_out[e] = 128 * s_pref[e];

    const int tile = blockIdx.x;
    if (tile >= s_pref[E]) return;   // block-uniform
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pref[mid] <= tile) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int tb = tile - s_pref[e];
    const int64_t pcol = (int64_t)128 * s_pref[e] + 128 * tb;
    if (pcol + 128 > a.P) return;
    const int32_t Te = a.offsets[e + 1] - a.offsets[e];
    const int n_in = min(128, Te - 128 * tb);
    const int64_t row0 = (int64_t)a.offsets[e] + 128 * tb;
    if (t < 128) {
        const int64_t lr = row0 + t;
        int32_t sr = -1;
        if (t < n_in && lr < a.R) {
            const int64_t v = a.row_map ? (int64_t)a.row_map[lr] : lr;
            if (v >= 0 && v < a.T_src) sr = (int32_t)v;
        }
        s_rows[t] = sr;
    }
    __syncthreads();
    // this CTA's column blocks
    const int ncb = (int)(a.C / 128);
    const int cb0 = (int)((int64_t)ncb * blockIdx.y / gridDim.y), cb1 = (int)((int64_t)ncb * (blockIdx.y + 1) / gridDim.y);
    // per thread: its 8 pieces' source rows are fixed for the tile
    const uint16_t* srcp[8];
    uint32_t nbytes[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int u = t + kColThreads * j;
        const int32_t sr = s_rows[u >> 4];
        srcp[j] = a.x + (sr >= 0 ? (int64_t)sr * a.C + (u & 15) * 8 : 0);
        nbytes[j] = sr >= 0 ? 16u : 0u;
    }
    // stage layout: word w of row r at word w ^ sw(r), sw(r) = 8 * ((r >> 5) & 3),
    // so the four token quarters a warp reads land on different banks
    auto issue = [&](int cb, int st) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int u = t + kColThreads * j;
            const int row = u >> 4, ch = u & 15;
            const int pw = (4 * ch) ^ (8 * ((row >> 5) & 3));
            cp_async16(fg8::tma::smem_u32(s_tile + st * kColTileBytes + row * 256 + pw * 4),
                       srcp[j] + (nbytes[j] ? (int64_t)cb * 128 : 0), nbytes[j]);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // warp wp owns column pairs 8 wp .. 8 wp + 7; lane = 8 q + pl: quarter q of
    // the tokens (32 each) of pair p = 8 wp + pl
    const int wp = t >> 5, lane = t & 31;
    const int q = lane >> 3, p = 8 * wp + (lane & 7);
    uint16_t* fix_list = reinterpret_cast<uint16_t*>(s_pref) + wp * kColFixCap;
    float2* col_sc = reinterpret_cast<float2*>(s_pref + 512) + wp * 8;
    if (cb0 < cb1) issue(cb0, 0);
    for (int cb = cb0; cb < cb1; ++cb) {
        const int st = (cb - cb0) & 1;
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();   // this block of rows has landed; the other stage is free
        if (cb + 1 < cb1) issue(cb + 1, st ^ 1);
        const int64_t col0 = (int64_t)cb * 128;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(s_tile + st * kColTileBytes);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = src[(32 * q + i) * 64 + (p ^ (8 * q))];
        // column maxima as a tree (4 independent chains), not one 32-long chain
        uint32_t mk[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 32; ++i) mk[i & 3] = __vmaxu2(mk[i & 3], w[i] & 0x7FFF7FFFu);
        uint32_t m = __vmaxu2(__vmaxu2(mk[0], mk[1]), __vmaxu2(mk[2], mk[3]));
        m = __vmaxu2(m, __shfl_xor_sync(kFull, m, 8));
        m = __vmaxu2(m, __shfl_xor_sync(kFull, m, 16));
        const float s0 = fg8::tile_scale(__uint_as_float((m & 0xFFFFu) << 16));
        const float s1 = fg8::tile_scale(__uint_as_float(m & 0xFFFF0000u));
        const fg8::QScale q0 = fg8::make_qscale(s0), q1 = fg8::make_qscale(s1);
        uint4 v0[4], v1[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            v0[g] = make_uint4(__byte_perm(w[8 * g + 0], w[8 * g + 1], 0x5410), __byte_perm(w[8 * g + 2], w[8 * g + 3], 0x5410),
                               __byte_perm(w[8 * g + 4], w[8 * g + 5], 0x5410), __byte_perm(w[8 * g + 6], w[8 * g + 7], 0x5410));
            v1[g] = make_uint4(__byte_perm(w[8 * g + 0], w[8 * g + 1], 0x7632), __byte_perm(w[8 * g + 2], w[8 * g + 3], 0x7632),
                               __byte_perm(w[8 * g + 4], w[8 * g + 5], 0x7632), __byte_perm(w[8 * g + 6], w[8 * g + 7], 0x7632));
        }
        // fast-path codes of all 8 groups; the groups whose brackets disagree
        // (bit g: column 2p, bit 4 + g: column 2p + 1) are redone exactly after
        // the stores, so the conversions themselves stay branch-free
        uint2 c0[4], c1[4];
        uint32_t redo = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            uint2 h0, h1;
            fg8::quant8_bracket(v0[g], q0, c0[g], h0);
            fg8::quant8_bracket(v1[g], q1, c1[g], h1);
            redo |= (uint32_t)(q0.exact || !fg8::bracket_agrees(c0[g], h0)) << g;
            redo |= (uint32_t)(q1.exact || !fg8::bracket_agrees(c1[g], h1)) << (4 + g);
        }
        uint8_t* d0 = a.xqT + (col0 + 2 * p) * a.P + pcol + 32 * q;
        uint8_t* d1 = d0 + a.P;
        reinterpret_cast<uint4*>(d0)[0] = make_uint4(c0[0].x, c0[0].y, c0[1].x, c0[1].y);
        reinterpret_cast<uint4*>(d0)[1] = make_uint4(c0[2].x, c0[2].y, c0[3].x, c0[3].y);
        reinterpret_cast<uint4*>(d1)[0] = make_uint4(c1[0].x, c1[0].y, c1[1].x, c1[1].y);
        reinterpret_cast<uint4*>(d1)[1] = make_uint4(c1[2].x, c1[2].y, c1[3].x, c1[3].y);
        if (q == 0)
            reinterpret_cast<float2*>(a.saT + (pcol / 128) * a.C + col0)[p] = make_float2(s0, s1);
        // exact codes of those groups from the staged words (this stage is not
        // refilled before the next iteration's barrier) over the fast-path
        // ones, shared out over the warp
        if (q == 0) col_sc[lane & 7] = make_float2(s0, s1);
        auto redo_group = [&](int owner, int b) {
            const int oq = owner >> 3, op = 8 * wp + (owner & 7), g = b & 3, hi = b >> 2;
            const uint32_t* wsrc = src + (32 * oq + 8 * g) * 64 + (op ^ (8 * oq));
            uint32_t wk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) wk[k] = wsrc[k * 64];
            const uint32_t sel = hi ? 0x7632u : 0x5410u;
            const uint4 v = make_uint4(__byte_perm(wk[0], wk[1], sel), __byte_perm(wk[2], wk[3], sel),
                                       __byte_perm(wk[4], wk[5], sel), __byte_perm(wk[6], wk[7], sel));
            const float2 sp = col_sc[owner & 7];
            const uint2 c = fg8::quant8_redo(v, fg8::make_qscale(hi ? sp.y : sp.x));
            *reinterpret_cast<uint2*>(a.xqT + (col0 + 2 * op + hi) * a.P + pcol + 32 * oq + 8 * g) = c;
        };
        if (!fg8::coop_redo(redo, fix_list, kColFixCap, redo_group)) {
            while (redo != 0u) {
                const int b = __ffs(redo) - 1;
                redo &= redo - 1u;
                redo_group(lane, b);
            }
            __syncwarp();
        }
    }
}

size_t ws_layout(int64_t E, size_t* off_totals, size_t* off_chunks);
inline void ws_layout_fwd(int64_t E, size_t* a, size_t* b) { ws_layout(E, a, b); }

// Cooperative launch of a permuting kernel (all CTAs resident: its grid
// barriers need that) on the workspace; the barrier word is cleared first.
fg8_status launch_permuting(const void* kern, RouteArgs& a, void* workspace, cudaStream_t st) {
    size_t off_tot, off_chk;
    ws_layout_fwd(a.E, &off_tot, &off_chk);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess ||
        per_sm < 1)
        return FG8_ERR_CUDA;
    int64_t G = (int64_t)per_sm * fg8h::num_sms();
    if (G > kMaxGrid) G = kMaxGrid;
    if (G > (a.T + 1) / 2) G = (a.T + 1) / 2;
    if (G < 1) G = 1;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return FG8_ERR_CUDA;
    a.bar = reinterpret_cast<uint32_t*>(ws);
    a.totals = reinterpret_cast<int32_t*>(ws + off_tot);
    a.chunk_counts = reinterpret_cast<int32_t*>(ws + off_chk);
    void* args[] = {&a};
    if (cudaLaunchCooperativeKernel(kern, dim3((unsigned)G), dim3(kThreads), args, 0, st) !=
        cudaSuccess)
        return FG8_ERR_CUDA;
    return fg8h::launch_status();
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
        if (K / 128 > INT32_MAX || (T + 127) / 128 > 65535 || T > INT32_MAX)
            return FG8_ERR_UNSUPPORTED;
        CUtensorMap m;
        if (!fg8h::make_tensor_map_2d(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, (uint64_t)T,
                                      (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
            return FG8_ERR_CUDA;
        if (cudaFuncSetAttribute(quant_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRowBoxBytes) != cudaSuccess)
            return FG8_ERR_CUDA;
        dim3 grid((unsigned)(K / 128), (unsigned)((T + 127) / 128));
        quant_rows<<<grid, kRowThreads, kRowBoxBytes, st>>>(m, T, K, xq, sa, dev_status);
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
        RouteArgs a = {};
        a.x = x; a.T = T; a.K = K; a.ids = topk_ids; a.k = k; a.E = E;
        a.xq = xq; a.sa = sa; a.row_token = row_token; a.token_row = token_row;
        a.offsets_out = offsets_out;
        a.status = dev_status;
        return launch_permuting((const void*)route_quant, a, workspace, st);
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
        ColArgs a;
        a.x = x; a.T_src = T; a.R = R; a.C = K; a.row_map = row_token; a.offsets = offsets_in; a.E = E; a.P = P;
        a.xqT = xqT; a.saT = saT; a.padoff_out = offsets_out; a.status = dev_status;
        if (cudaFuncSetAttribute(colwise_tiles, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(2 * kColTileBytes)) != cudaSuccess)
            return FG8_ERR_CUDA;
        dim3 grid((unsigned)max_tiles, (unsigned)kColGroups);
        colwise_tiles<<<grid, kColThreads, 2 * kColTileBytes, st>>>(a);
        return fg8h::launch_status();
    }
    return FG8_ERR_INVALID_ARG;
}

extern "C" fg8_status fg8_route_quantize_act(const float* logits, const float* bias,
                                             const uint16_t* x, int64_t T, int64_t K, int k, int E,
                                             int32_t* topk_ids, float* affinity, uint8_t* xq,
                                             float* sa, int32_t* row_token, int32_t* token_row,
                                             int32_t* offsets_out, void* workspace, size_t ws_bytes,
                                             int32_t* dev_status, fg8_stream_t stream) {
    cudaStream_t st = (cudaStream_t)stream;
    if (T < 0 || K < 128 || K % 128 || E < 1 || E > 1024 || k < 1 || k > fg8::kRouteMaxK || k > E)
        return FG8_ERR_INVALID_ARG;
    if (!offsets_out) return FG8_ERR_INVALID_ARG;
    if (T == 0)
        return cudaMemsetAsync(offsets_out, 0, sizeof(int32_t) * ((size_t)E + 1), st) == cudaSuccess
                   ? FG8_OK : FG8_ERR_CUDA;
    if (!logits || !bias || !x || !topk_ids || !affinity || !xq || !sa || !row_token ||
        !token_row || !workspace)
        return FG8_ERR_INVALID_ARG;
    if (!fg8h::aligned16(x) || !fg8h::aligned16(xq) || !fg8h::aligned16(workspace) ||
        ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(bias) |
          reinterpret_cast<uintptr_t>(affinity) | reinterpret_cast<uintptr_t>(sa)) & 3))
        return FG8_ERR_INVALID_ARG;
    if (T * k > (int64_t)INT32_MAX || T > INT64_MAX / E) return FG8_ERR_UNSUPPORTED;
    size_t off_tot, off_chk;
    if (ws_bytes < ws_layout(E, &off_tot, &off_chk)) return FG8_ERR_INVALID_ARG;
    RouteArgs a = {};
    a.x = x; a.T = T; a.K = K; a.ids = topk_ids; a.k = k; a.E = E;
    a.xq = xq; a.sa = sa; a.row_token = row_token; a.token_row = token_row;
    a.offsets_out = offsets_out;
    a.status = dev_status;
    a.logits = logits; a.bias = bias; a.ids_out = topk_ids; a.affinity = affinity;
    const void* kern = E <= 64    ? (const void*)route_topk_quant<2>
                       : E <= 128 ? (const void*)route_topk_quant<4>
                       : E <= 256 ? (const void*)route_topk_quant<8>
                       : E <= 512 ? (const void*)route_topk_quant<16>
                                  : (const void*)route_topk_quant<32>;
    return launch_permuting(kern, a, workspace, st);
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
// it, keyed by the unique id of the device's current context: if the context
// is replaced (cudaDeviceReset, or the primary context released and created
// again), the module is loaded anew, the array may move, and the next call
// looks the address up again.  That first call (and the first after such a
// replacement) should therefore come before any stream capture.

namespace {

constexpr int kNoAllocMaxExperts = 256;
constexpr size_t kNoAllocScratchBytes =
    256 + 4 * (size_t)kNoAllocMaxExperts + (size_t)kMaxGrid * kNoAllocMaxExperts * 4;  // ~1 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
struct NoallocCache {
    unsigned long long ctx_id;   // unique id of the context the address belongs to
    void* addr;
};
NoallocCache g_noalloc_cache[kMaxDevices];
std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context (ids are never reused), or
// 0 if there is none yet or the driver cannot tell.
unsigned long long current_context_id() {
    static const CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array in the current device's current context.
fg8_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FG8_ERR_CUDA;
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocCache& c = g_noalloc_cache[dev];
    if (id != 0 && c.ctx_id == id && c.addr != nullptr) {
        *out = c.addr;
        return FG8_OK;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return FG8_ERR_CUDA;
    c.ctx_id = current_context_id();   // the lookup has made the context current
    c.addr = p;
    *out = p;
    return FG8_OK;
}

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
    void* scratch = nullptr;
    const fg8_status found = noalloc_scratch(&scratch);
    if (found != FG8_OK) return found;
    // the permuting entry point clears the barrier word on every call; the
    // per-chunk counts and totals are fully written before they are read
    return fg8_quantize_act(x, T, K, topk_ids, k, E, nullptr, FG8_ROWWISE, xq, sa, row_token,
                            token_row, offsets_out, nullptr, nullptr, scratch,
                            kNoAllocScratchBytes, dev_status, stream);
}
