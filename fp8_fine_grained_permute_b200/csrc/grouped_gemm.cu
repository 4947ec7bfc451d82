// grouped_gemm.cu -- grouped FP8 GEMM with fine-grained scales on tcgen05.
//
// Computes, for every expert e (DeepSeek-V3 summary sec. 2.2: most GEMMs in
// FP8 with 1x128 / 128x128 scaling and high-precision accumulation; Kanana-2
// deep dive, devday.kr, FP8 paragraph):
//     out[r][n] = sum_kb  sA(r,kb) * sB(n,kb) * sum_{k in block kb} A[r][k] * B[n][k]
// The scales are arbitrary fp32 values, so they cannot be folded into the
// tensor-core instruction (its block-scaled form takes power-of-two scales at
// 32-element granularity).  Instead each 128-wide K block is multiplied on the
// tensor core into its own TMEM partial (fp32), and the promotion warps add
// partial * sA * sB into fp32 accumulators held in registers: DeepSeek-V3's
// promotion to CUDA cores, with the partial sums living in TMEM.
//
// CTA = one persistent worker per SM, 12 warps (setmaxnreg gives the control
// warpgroup 40 registers a thread and the promotion warpgroups 232):
//   warp 0      TMA producer: A tile 128x128 B and B tile 256x128 B per K block
//               into a 4-stage (row-grouped) or 3-stage (contraction-grouped)
//               ring of 48 KB stages, 128-byte swizzle; contraction-grouped, it
//               also bulk-copies the K block's 128 + 256 scales into a slot ring.
//   warp 1      TMEM allocator + MMA issuer: 4 x tcgen05.mma (M=128, N=256,
//               K=32, E4M3 x E4M3 -> f32) per K block into one of two TMEM
//               partial buffers (2 x 256 columns); tcgen05.commit frees the smem
//               stage and publishes the partial.
//   warps 2, 3  idle.
//   warps 4..11 promotion + epilogue: two warpgroups, one per 128-column half.
//               Row-grouped (one scale per row and K block): thread = one output
//               row, 32x32b loads.  Contraction-grouped (a scale per row and per
//               column): 16x256b loads, thread = 4 rows x 32 columns, so it reads
//               16 column-scale pairs instead of 128 scales per K block.
//               acc = fma(partial, sA*sB, acc), then release the buffer; after
//               the last K block the tile goes out through shared memory (8-row
//               x 64-byte stores, or 32x32 fp32 boxes drained by TMA stores).
// Tiles are 128 rows x 256 columns; the tile list (expert, m-tile, n-tile) is
// rebuilt on the device from the expert offsets (kept in shared memory), so
// offsets never travel to the host.  Zero-row experts have no tiles
// (row-grouped mode); in the contraction-grouped mode an expert with no tokens
// writes zeros.
//
// Gate/up mode (row-grouped, fg8_grouped_gemm_swiglu_quant): a tile is 128
// rows x 128 output columns whose 256-row B operand is the expert's gate block
// and up block for those columns (two 128-row TMA boxes), so warpgroup 0
// accumulates the gate and warpgroup 1 the up projection; after the last K
// block the up values are handed to the gate warps through TMEM and the
// epilogue writes silu(gate) * up as E4M3 codes with one scale per 1x128 tile.
//
// Every mbarrier wait is bounded (FG8_ERR_TIMEOUT in *status, then the roles
// wind down and TMEM is released); the kernel never traps.
#include <cuda.h>

#include "fg8_common.cuh"
#include "fg8_tma.cuh"

namespace {

using namespace fg8::tma;

// 128 x 256 tiles: N = 256 is the widest single-CTA tcgen05.mma.  Narrower
// tiles do not pay here: 128 x 128 tiles with four TMEM buffers ran at 0.6x the
// throughput, because the promotion's fixed cost per K block (waits, fences,
// buffer release, scale loads) is then spread over half the work, although an
// N = 128 MMA on its own takes half the time of an N = 256 one.
constexpr int BM = 128, BN = 256, BK = 128;
constexpr uint32_t kABytes = BM * BK;              // 16 KB
constexpr uint32_t kBBytes = BN * BK;              // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kCtrlWarps = 4;                      // warpgroup 0: TMA, MMA, 2 idle warps
// Promotion warps: two warpgroups of 128 columns each, in both modes.  (Four
// warpgroups of 64 columns, at 112 registers, were measured slower for the
// row-grouped mode: 2.85 -> 3.94 ms on the DeepSeek-shaped fprop, so the packed
// FMA work, not latency, bounds the promotion there.)
// Register split (setmaxnreg): the control warpgroup gives registers back and
// the promotion warpgroups take them.  The split must not exceed what the CTA
// was launched with (threads x registers per thread), or the increase would
// wait forever; the host refuses to launch unless the compiled kernel has
// >= kLaunchRegs.
template <bool kGroupK>
struct Warps {
    static constexpr int kEpiWarps = 8;
    static constexpr int kThreads = 32 * (kCtrlWarps + kEpiWarps);   // 384
    static constexpr int kCols = BN / (kEpiWarps / 4);               // columns per promotion warp
    static constexpr int kCtrlRegs = 40;
    static constexpr int kEpiRegs = 232;
    static constexpr int kLaunchRegs = 168;
    static_assert(32 * kCtrlWarps * kCtrlRegs + 32 * kEpiWarps * kEpiRegs <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static_assert(kLaunchRegs * kThreads <= 65536, "launch allocation exceeds the register file");
};
constexpr int kMaxE = 1024;
constexpr uint32_t kTmemCols = 512;                // two partial buffers of BN columns

// tcgen05 instruction descriptor (kind::f8f6f4): D = f32 (bits 4-5 = 1),
// A = B = E4M3 (format 0), both K-major, N >> 3 in bits 17-22, M >> 4 in 24-28.
constexpr uint32_t kIdesc =
    (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// row-grouped epilogue staging: per promotion warp 32 rows x 16 words (+4 padding)
constexpr int kStageWords = 20;
constexpr uint32_t kStagePerWarp = 32 * kStageWords * 4;         // 2560 bytes
// contraction-grouped epilogue: per promotion warp two 32 x 32 fp32 boxes
// (4 KB each, 128-byte swizzle) drained by TMA stores
constexpr uint32_t kBoxBytes = 32 * 32 * 4;
constexpr uint32_t kTmaStagePerWarp = 2 * kBoxBytes;
// contraction-grouped mode: per K block the producer also copies the 128 row
// scales of A and the 256 column scales of B into a ring of slots.  The slot of
// K block n is rewritten for block n + kScaleSlots.  The producer loads block n
// only after the MMA of block n - kStages released that stage, and that MMA
// started only after the promotion of block n - kStages - 2 released its TMEM
// buffer (having read its scales first).  So kScaleSlots >= kStages + 2 slots
// are never rewritten before their reader is done.
constexpr uint32_t kScaleSlotBytes = 4 * (BM + BN);            // 1536

constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// contraction-grouped mode: tiles are handed out at run time.  The producer
// takes the next tile number from a counter in the caller's workspace (zeroed
// on the stream before the launch), decodes it and publishes what the other roles need (K blocks, first output
// row and column) through a ring of kTileRing shared slots; the MMA thread and
// the promotion warps read the ring.  Experts with few tokens are output-bound
// (a 128 KB fp32 tile per 128x256 block) and experts with many are math-bound,
// so the order interleaves the tiles of kMix experts of different sizes (one
// from each size quantile) to keep both busy; within an expert, consecutive
// tiles share their A rows.
constexpr int kTileRing = 8;
constexpr int kMix = 4;
// Caller workspace of the contraction-grouped mode (zeroed before each launch):
// word 0 is the tile ticket counter, word 1 counts the producers that have
// finished, so the last one can check the ticket count (a workspace shared by
// overlapping launches breaks it, and is reported instead of passing
// unnoticed).
constexpr size_t kGroupKWorkspace = 16;

// shared memory map (offsets from a 1024-byte aligned base), per mode
template <bool kGroupK>
struct Layout {
    static constexpr int kStages = kGroupK ? 3 : 4;    // short K loops need fewer
    static constexpr int kScaleSlots = kStages + 2;
    static constexpr uint32_t kOffStages = 0;
    static constexpr uint32_t kOffBars = kStages * kStageBytes;
    // full, empty, tfull, tempty, drain, then the tile ring (contraction-
    // grouped) or the gate/up epilogue's exchange barriers (row-grouped)
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1 + (kGroupK ? 2 * kTileRing : 8);
    static constexpr uint32_t kOffMisc = kOffBars + 8 * kNumBars;   // tmem slot, abort flag
    static constexpr uint32_t kOffRing = align_up(kOffMisc + 16, 16);  // int4 [kTileRing]
    // row-grouped: tiles per expert, exclusive prefix; contraction-grouped:
    // the experts in processing order
    static constexpr uint32_t kOffTiles = kOffRing + 16 * kTileRing;   // int32 [kMaxE + 1]
    static constexpr uint32_t kOffOffs = kOffTiles + 4 * (kMaxE + 4);   // int32 [kMaxE + 1]
    static constexpr uint32_t kOffWarp = kOffOffs + 4 * (kMaxE + 4);    // int32 [36]
    static constexpr uint32_t kOffStage = align_up(kOffWarp + 4 * 36, kGroupK ? 1024 : 16);
    static constexpr uint32_t kStageAll =
        Warps<kGroupK>::kEpiWarps * (kGroupK ? kTmaStagePerWarp : kStagePerWarp);
    static constexpr uint32_t kOffScales = kOffStage + kStageAll;
    // contraction-grouped: the scale slots; row-grouped: the gate/up
    // epilogue's row maxima, [TMEM buffer][warpgroup][row]
    static constexpr uint32_t kSmemBytes =
        kOffScales + (kGroupK ? kScaleSlots * kScaleSlotBytes : 2 * 2 * BM * 4) + 1024;   // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kOffStage % 16 == 0 && (kStageWords * 4) % 16 == 0, "16-byte staging");
};

struct GemmArgs {
    const float* sa;
    const float* sb;
    const int32_t* offsets;
    int64_t M_total;
    int N, K, E;
    int mode;       // FG8_GROUP_M / FG8_GROUP_K
    int out_f32;
    void* out;
    int32_t* status;
    unsigned int* ws;         // contraction-grouped: zeroed workspace words (see kGroupKWorkspace)
    // row-grouped gate/up mode: B holds [gate; up] (N = 2 I rows per expert),
    // out = E4M3 codes of h = silu(gate) * up [M_total][I], out_scale = their
    // 1x128 scales [I/128][M_total]
    int swiglu;
    float* out_scale;
    // row-grouped combine mode: out = fp32 [T][N] token rows, each routed row
    // added with its gate weight: row_tok[r], row_w[r] (fg8_grouped_gemm_combine)
    const int32_t* row_tok;
    const float* row_w;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

// K-major operand tile in shared memory, 128-byte rows, 128-byte swizzle:
// 8-row atoms 1024 bytes apart (stride byte offset), descriptor version 1.
FG8_DEV uint64_t smem_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;                  // leading byte offset (unused with this swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset
    d |= (uint64_t)1 << 46;                  // descriptor version
    d |= (uint64_t)2 << 61;                  // SWIZZLE_128B
    return d;
}

FG8_DEV void mma_e4m3(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

FG8_DEV void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

FG8_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FG8_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// out[0..3] += (x, y, z, w), one 16-byte fp32 reduction in L2 (16-byte aligned)
FG8_DEV void red_add_v4(float* out, float x, float y, float z, float w) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(out), "f"(x), "f"(y), "f"(z), "f"(w)
                 : "memory");
}

// 32 lanes x 64 consecutive fp32 columns of TMEM -> 64 registers per thread,
// waited for inside the same asm statement (the outputs exist only after
// tcgen05.wait::ld, so no use can be scheduled before the wait).
FG8_DEV void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// Two 16-lane halves' worth of the 16x256b shape, 8 repetitions: thread t of
// the warp gets, for repetition j, the fp32 values at (lane t/4, column
// 8j + 2(t%4) + {0,1}) in r[4j], r[4j+1] and at (lane t/4 + 8, same columns)
// in r[4j+2], r[4j+3], lanes counted from the address's lane field.  Waited
// for inside the statement.
FG8_DEV void tmem_ld16x256_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 64 fp32 values of this thread -> 32 lanes x 64 consecutive TMEM columns
// (the 32x32b shape: a thread's values go to its own lane).  Completed by
// tcgen05.wait::st.
FG8_DEV void tmem_st64(uint32_t taddr, const float2* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n"
                 ::"r"(taddr), "r"(__float_as_uint(v[0].x)), "r"(__float_as_uint(v[0].y)), "r"(__float_as_uint(v[1].x)), "r"(__float_as_uint(v[1].y)), "r"(__float_as_uint(v[2].x)), "r"(__float_as_uint(v[2].y)), "r"(__float_as_uint(v[3].x)), "r"(__float_as_uint(v[3].y)), "r"(__float_as_uint(v[4].x)), "r"(__float_as_uint(v[4].y)), "r"(__float_as_uint(v[5].x)), "r"(__float_as_uint(v[5].y)), "r"(__float_as_uint(v[6].x)), "r"(__float_as_uint(v[6].y)), "r"(__float_as_uint(v[7].x)), "r"(__float_as_uint(v[7].y)), "r"(__float_as_uint(v[8].x)), "r"(__float_as_uint(v[8].y)), "r"(__float_as_uint(v[9].x)), "r"(__float_as_uint(v[9].y)), "r"(__float_as_uint(v[10].x)), "r"(__float_as_uint(v[10].y)), "r"(__float_as_uint(v[11].x)), "r"(__float_as_uint(v[11].y)), "r"(__float_as_uint(v[12].x)), "r"(__float_as_uint(v[12].y)), "r"(__float_as_uint(v[13].x)), "r"(__float_as_uint(v[13].y)), "r"(__float_as_uint(v[14].x)), "r"(__float_as_uint(v[14].y)), "r"(__float_as_uint(v[15].x)), "r"(__float_as_uint(v[15].y)), "r"(__float_as_uint(v[16].x)), "r"(__float_as_uint(v[16].y)), "r"(__float_as_uint(v[17].x)), "r"(__float_as_uint(v[17].y)), "r"(__float_as_uint(v[18].x)), "r"(__float_as_uint(v[18].y)), "r"(__float_as_uint(v[19].x)), "r"(__float_as_uint(v[19].y)), "r"(__float_as_uint(v[20].x)), "r"(__float_as_uint(v[20].y)), "r"(__float_as_uint(v[21].x)), "r"(__float_as_uint(v[21].y)), "r"(__float_as_uint(v[22].x)), "r"(__float_as_uint(v[22].y)), "r"(__float_as_uint(v[23].x)), "r"(__float_as_uint(v[23].y)), "r"(__float_as_uint(v[24].x)), "r"(__float_as_uint(v[24].y)), "r"(__float_as_uint(v[25].x)), "r"(__float_as_uint(v[25].y)), "r"(__float_as_uint(v[26].x)), "r"(__float_as_uint(v[26].y)), "r"(__float_as_uint(v[27].x)), "r"(__float_as_uint(v[27].y)), "r"(__float_as_uint(v[28].x)), "r"(__float_as_uint(v[28].y)), "r"(__float_as_uint(v[29].x)), "r"(__float_as_uint(v[29].y)), "r"(__float_as_uint(v[30].x)), "r"(__float_as_uint(v[30].y)), "r"(__float_as_uint(v[31].x)), "r"(__float_as_uint(v[31].y))
                 : "memory");
}

// silu(g) * u = g / (1 + e^-g) * u, fast exponential and division (the
// result is quantized to E4M3 next; both are within a few fp32 ulps)
FG8_DEV float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

FG8_DEV uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------
// tile schedule
// ---------------------------------------------------------------------------

struct Tile {
    int e;
    int rows_valid;     // rows of the tile that belong to the expert
    int n0;             // first output column
    int kx0;            // first contraction column of the operands
    int nkb;            // 128-wide contraction blocks
    int64_t rowA;       // first operand-A row
    int64_t rowB;       // first operand-B row
    int64_t rowB2;      // gate/up mode: first row of the up block (second half of B)
    int64_t out_row0;   // first output row
};

// Row-grouped: s_tiles is the exclusive prefix of tiles per expert (E + 1
// entries), s_off the expert offsets, both in shared memory.  A thread's tiles only increase, so
// the expert of its previous tile (e_hint) starts the search.
FG8_DEV Tile decode_tile(int tile, const int32_t* s_tiles, const int32_t* s_off, const GemmArgs& a,
                         int nt, int& e_hint) {
    int lo = e_hint;   // s_tiles[lo] <= tile; find the largest such e
    if (s_tiles[lo + 1] <= tile) {
        int hi = a.E;  // s_tiles[E] = total > tile
        ++lo;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_tiles[mid] <= tile) lo = mid; else hi = mid;
        }
    }
    e_hint = lo;
    Tile T;
    T.e = lo;
    const int local = tile - s_tiles[lo];
    const int mt = local / nt, ntile = local - mt * nt;
    // gate/up mode: a tile is 128 output columns, its B is gate block + up block
    T.n0 = a.swiglu ? ntile * 128 : ntile * BN;
    const int32_t o0 = s_off[lo], o1 = s_off[lo + 1];
    T.rowA = (int64_t)o0 + (int64_t)mt * BM;
    // rows past M_total (offsets inconsistent with the buffers) are never touched
    T.rows_valid = (int)max((int64_t)0, min((int64_t)min(BM, (o1 - o0) - mt * BM),
                                            a.M_total - T.rowA));
    T.kx0 = 0;
    T.nkb = a.K / BK;
    T.rowB = (int64_t)lo * a.N + T.n0;
    T.rowB2 = (int64_t)lo * a.N + a.N / 2 + T.n0;
    T.out_row0 = T.rowA;
    return T;
}

// Contraction-grouped: g -> (expert, m-tile, n-tile).  s_order lists the experts
// in processing order, in groups of `mix` whose tiles alternate; every expert
// has tpe tiles.
FG8_DEV Tile decode_tile_k(int g, const int32_t* s_order, const int32_t* s_off, const GemmArgs& a,
                           int nt, int tpe, int mix) {
    const int grp = g / (mix * tpe);
    const int rem = g - grp * mix * tpe;
    const int e = s_order[grp * mix + rem % mix];
    const int local = rem / mix;
    const int mt = local / nt, ntile = local - mt * nt;
    Tile T;
    T.e = e;
    T.n0 = ntile * BN;
    const int32_t o0 = s_off[e], o1 = s_off[e + 1];
    T.rowA = (int64_t)mt * BM;
    T.rows_valid = BM;
    // contraction range clamped to the operands' width
    T.kx0 = min(max(o0, 0), a.K) & ~(BK - 1);
    T.nkb = max(0, min(o1, a.K) - T.kx0) / BK;
    T.rowB = T.n0;
    T.rowB2 = -1;
    T.out_row0 = (int64_t)e * a.M_total + T.rowA;
    return T;
}

// K blocks of expert e in the contraction-grouped mode (as decode_tile_k)
FG8_DEV int expert_kblocks(const int32_t* s_off, int e, int K) {
    const int kx0 = min(max(s_off[e], 0), K) & ~(BK - 1);
    return max(0, min(s_off[e + 1], K) - kx0) / BK;
}

// tile ring: the producer publishes, the other roles take (bounded waits).
// An entry is {K blocks, first output row, first output column, 0}; K blocks
// -1 ends the stream.
struct TileRing {
    int4* slots;
    uint32_t full0, empty0;   // mbarrier addresses of slot 0
    uint32_t slot = 0, phase = 0;
    FG8_DEV void advance() {
        if (++slot == kTileRing) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

FG8_DEV bool ring_wait_free(TileRing& R, volatile int* abort_flag, int32_t* status) {
    return mbar_wait(R.empty0 + 8u * R.slot, R.phase ^ 1u, abort_flag, status);
}

FG8_DEV void ring_publish(TileRing& R, int4 v) {
    asm volatile("st.shared.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(R.slots + R.slot)),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
    mbar_arrive(R.full0 + 8u * R.slot);   // release: the entry is visible to the takers
    R.advance();
}

// whole_warp: every lane of the warp calls this (lane 0 releases the slot);
// otherwise a single thread does.
FG8_DEV bool ring_take(TileRing& R, bool whole_warp, int4& v, volatile int* abort_flag,
                       int32_t* status) {
    if (!mbar_wait(R.full0 + 8u * R.slot, R.phase, abort_flag, status)) return false;
    asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(R.slots + R.slot))
                 : "memory");
    if (whole_warp) __syncwarp();
    if (!whole_warp || (threadIdx.x & 31) == 0) mbar_arrive(R.empty0 + 8u * R.slot);
    R.advance();
    return true;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

template <bool kGroupK, bool kSwiglu = false, bool kCombine = false>
__global__ void __launch_bounds__(Warps<kGroupK>::kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const GemmArgs a) {
    using L = Layout<kGroupK>;
    using Wp = Warps<kGroupK>;
    constexpr int kThreads = Wp::kThreads, kEpiWarps = Wp::kEpiWarps, kCols = Wp::kCols;
    constexpr int kStages = L::kStages;
    constexpr int kScaleSlots = L::kScaleSlots;
    constexpr uint32_t kOffStages = L::kOffStages, kOffBars = L::kOffBars, kOffMisc = L::kOffMisc;
    constexpr uint32_t kOffTiles = L::kOffTiles, kOffWarp = L::kOffWarp, kOffStage = L::kOffStage;
    constexpr uint32_t kOffScales = L::kOffScales;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kOffBars;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
    // row-grouped gate/up epilogue: per TMEM buffer and warpgroup, one barrier
    // for the half of the accumulators handed over and one for the row maxima
    // (4 arrivals each).  A buffer is reused only after both warpgroups have
    // released it, which they do after their waits, so no exchange barrier
    // can complete twice before its waiters have seen it.
    auto xchg_bar = [&](uint32_t b, int g) { return bar0 + 8u * (2 * kStages + 5 + 2 * b + g); };
    auto amax_bar = [&](uint32_t b, int g) { return bar0 + 8u * (2 * kStages + 9 + 2 * b + g); };
    const uint32_t ring_full0 = bar0 + 8u * (2 * kStages + 5);
    const uint32_t ring_empty0 = ring_full0 + 8u * kTileRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + kOffTiles);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + L::kOffOffs);
    int32_t* s_warp = reinterpret_cast<int32_t*>(smem + kOffWarp);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = (!kGroupK && kSwiglu) ? a.N / 256 : (a.N + BN - 1) / BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        if (!kGroupK)
            for (int b = 0; b < 2; ++b)
                for (int g = 0; g < 2; ++g) {
                    mbar_init(xchg_bar(b, g), kEpiWarps / 2);
                    mbar_init(amax_bar(b, g), kEpiWarps / 2);
                }
        if (kGroupK) {
            for (int i = 0; i < kTileRing; ++i) {
                mbar_init(ring_full0 + 8u * i, 1);
                mbar_init(ring_empty0 + 8u * i, 1 + kEpiWarps);   // MMA thread + promotion warps
            }
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int e = threadIdx.x; e <= a.E; e += kThreads) s_off[e] = a.offsets[e];
    const int mix = (kGroupK && a.E % kMix == 0) ? kMix : 1;
    const int tpe = (int)(a.M_total / BM) * nt;   // contraction-grouped: tiles per expert
    if (!kGroupK) {
        // tiles per expert -> exclusive prefix (in place)
        for (int e = threadIdx.x; e < a.E; e += kThreads)
            s_tiles[e] = (max(0, a.offsets[e + 1] - a.offsets[e]) + BM - 1) / BM * nt;
        __syncthreads();
        fg8::block_exclusive_scan(s_tiles, s_tiles, a.E, s_warp);
    } else {
        // processing order: rank the experts by K blocks (descending, ties by
        // id); group i takes ranks i, i + E/mix, i + 2E/mix, ... (one per size
        // quantile)
        __syncthreads();
        const int ng = a.E / mix;
        for (int e = threadIdx.x; e < a.E; e += kThreads) {
            const int ke = expert_kblocks(s_off, e, a.K);
            int rank = 0;
            for (int f = 0; f < a.E; ++f) {
                const int kf = expert_kblocks(s_off, f, a.K);
                rank += (kf > ke) || (kf == ke && f < e);
            }
            s_tiles[(rank % ng) * mix + rank / ng] = e;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = kGroupK ? a.E * tpe : s_tiles[a.E];
    TileRing ring;
    ring.slots = reinterpret_cast<int4*>(smem + L::kOffRing);
    ring.full0 = ring_full0;
    ring.empty0 = ring_empty0;

    if (warp < kCtrlWarps) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Wp::kCtrlRegs));
      if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            uint32_t stage = 0, phase = 0, sc = 0;
            int e_hint = 0;
            bool ok = true;
            for (int tile = (int)blockIdx.x - (int)gridDim.x;;) {
                Tile T;
                if (kGroupK) {
                    if (!ring_wait_free(ring, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tile = (int)atomicAdd(a.ws, 1u);
                    if (tile >= total || tile < 0) {
                        ring_publish(ring, make_int4(-1, 0, 0, 0));
                        break;
                    }
                    T = decode_tile_k(tile, s_tiles, s_off, a, nt, tpe, mix);
                    ring_publish(ring, make_int4(T.nkb, (int)T.out_row0, T.n0, 0));
                } else {
                    if ((tile += gridDim.x) >= total) break;
                    T = decode_tile(tile, s_tiles, s_off, a, nt, e_hint);
                }
                for (int kb = 0; kb < T.nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sA = sbase + kOffStages + stage * kStageBytes;
                    if (kGroupK) {
                        const int kbg = T.kx0 / BK + kb;
                        const uint32_t sb_bytes = 4u * (uint32_t)min(BN, a.N - T.n0);
                        const uint32_t slot = sbase + kOffScales + (sc % kScaleSlots) * kScaleSlotBytes;
                        mbar_arrive_expect_tx(full_bar(stage), kStageBytes + 4 * BM + sb_bytes);
                        bulk_load(slot, a.sa + (int64_t)kbg * a.M_total + T.rowA, 4 * BM, full_bar(stage));
                        bulk_load(slot + 4 * BM, a.sb + (int64_t)kbg * a.N + T.n0, sb_bytes, full_bar(stage));
                        ++sc;
                    } else {
                        mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
                    }
                    if (kGroupK) {
                        // the operands stay in L2 for the expert's other tiles
                        // while the fp32 output streams past them (evict-first)
                        const uint64_t keep = l2_policy_evict_last();
                        tma_load_2d_hint(&tmA, sA, full_bar(stage), T.kx0 + kb * BK, (int)T.rowA, keep);
                        tma_load_2d_hint(&tmB, sA + kABytes, full_bar(stage), T.kx0 + kb * BK, (int)T.rowB,
                                         keep);
                    } else if (kSwiglu) {   // B map boxes are 128 rows here
                        tma_load_2d(&tmA, sA, full_bar(stage), T.kx0 + kb * BK, (int)T.rowA);
                        tma_load_2d(&tmB, sA + kABytes, full_bar(stage), T.kx0 + kb * BK, (int)T.rowB);
                        tma_load_2d(&tmB, sA + kABytes + kBBytes / 2, full_bar(stage), T.kx0 + kb * BK,
                                    (int)T.rowB2);
                    } else {
                        tma_load_2d(&tmA, sA, full_bar(stage), T.kx0 + kb * BK, (int)T.rowA);
                        tma_load_2d(&tmB, sA + kABytes, full_bar(stage), T.kx0 + kb * BK, (int)T.rowB);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            if (!ok) {
                // let copies already issued land before the CTA winds down
                const uint32_t last = (stage + kStages - 1) % kStages;
                const uint32_t lp = stage == 0 ? (phase ^ 1u) : phase;
                const uint64_t t0 = fg8::globaltimer_ns();
                while (!mbar_try_wait(full_bar(last), lp) &&
                       fg8::globaltimer_ns() - t0 < 100000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            uint32_t stage = 0, phase = 0, buf = 0, bphase = 0;
            bool ok = true;
            for (int tile = (int)blockIdx.x - (int)gridDim.x;;) {
                int nkb;
                if (kGroupK) {
                    int4 v;
                    if (!ring_take(ring, false, v, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    if (v.x < 0) break;
                    nkb = v.x;
                } else {
                    if ((tile += gridDim.x) >= total) break;
                    nkb = a.K / BK;   // every row-grouped tile spans the whole contraction
                }
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(tempty_bar(buf), bphase ^ 1u, abort_flag, a.status) ||
                        !mbar_wait(full_bar(stage), phase, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sA = sbase + kOffStages + stage * kStageBytes;
                    const uint32_t d = tmem_base + buf * BN;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_e4m3(d, smem_desc(sA + 32 * kk), smem_desc(sA + kABytes + 32 * kk),
                                 kk > 0 ? 1u : 0u);
                    mma_commit(empty_bar(stage));
                    mma_commit(tfull_bar(buf));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    buf ^= 1u;
                    if (buf == 0) bphase ^= 1u;
                }
                if (!ok) break;
            }
            // all MMAs issued by this thread are complete once drain_bar flips
            mma_commit(drain_bar);
            const uint64_t t0 = fg8::globaltimer_ns();
            while (!mbar_try_wait(drain_bar, 0) && fg8::globaltimer_ns() - t0 < 100000000ull) {
            }

        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Wp::kEpiRegs));
        // ---------------------------------------------------- promotion + epilogue
        const int ep = warp - kCtrlWarps;
        const int grp = ep >> 2;             // kCols-column group of the tile
        const int quarter = warp & 3;        // TMEM lane quarter this warp may access
        const int r = 32 * quarter + lane;   // tile row owned by this thread (row-grouped)
        const int g4 = lane >> 2, c2 = 2 * (lane & 3);   // 16x256b position (contraction-grouped)
        const int NB = a.N / 128, KBt = a.K / BK;
        uint32_t buf = 0, bphase = 0, sc = 0;
        uint32_t nbox = 0;    // TMA-store boxes issued by this warp (contraction-grouped)
        uint32_t xphase = 0;  // gate/up epilogue: bit b = phase of buffer b's exchange barriers
        int e_hint = 0;
        bool ok = true;
        // row-grouped mode: the scales of the next K block are loaded while this
        // one is promoted, and during a tile's last block those of the next
        // tile's first block, so no tile starts by waiting for a global load
        // (two blocks ahead measured slower in the full step: it costs the
        // promotion a spilled register)
        float sa_n = 0.f, sb_n = 0.f;
        bool next_loaded = false;
        // where a row-grouped tile's scales are, for this thread
        auto scale_ptrs = [&](const Tile& T, const float*& sap, const float*& sbp, bool& rok, bool& cok) {
            rok = r < T.rows_valid;
            const int c0 = T.n0 + kCols * grp;
            cok = kSwiglu || c0 < a.N;
            // gate/up mode: both halves cover output columns n0..n0+127; the
            // second half's B rows (and block scales) are the up block
            const int bcol = kSwiglu ? (grp == 0 ? T.n0 : a.N / 2 + T.n0) : c0;
            sap = a.sa + T.rowA + r;
            sbp = a.sb + ((int64_t)T.e * NB + bcol / 128) * KBt;
        };
        for (int tile = (int)blockIdx.x - (int)gridDim.x;;) {
            int4 v = make_int4(0, 0, 0, 0);
            if (kGroupK) {
                if (!ring_take(ring, true, v, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                if (v.x < 0) break;
            } else if ((tile += gridDim.x) >= total) {
                break;
            }
            float2 acc[kCols / 2];   // row-grouped: columns 2i, 2i + 1 of this thread's group
#pragma unroll
            for (int i = 0; i < kCols / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            // Only what the K loop and the epilogue need stays live (registers
            // are the promotion's limit); output rows fit in 32 bits (checked
            // on the host).
            int nkb, rows_valid, out_row0, col0;
            bool row_ok, col_ok;
            const float* sa_p;
            const float* sb_p;
            if (kGroupK) {
                nkb = v.x;
                rows_valid = BM;
                out_row0 = v.y;
                row_ok = true;
                col0 = v.z + kCols * grp;
                col_ok = col0 < a.N;
                sa_p = sb_p = nullptr;
            } else {
                const Tile T = decode_tile(tile, s_tiles, s_off, a, nt, e_hint);
                nkb = T.nkb;
                rows_valid = T.rows_valid;
                out_row0 = (int)T.out_row0;
                col0 = kSwiglu ? T.n0 : T.n0 + kCols * grp;
                scale_ptrs(T, sa_p, sb_p, row_ok, col_ok);
                if (!next_loaded) {
                    sa_n = (row_ok && nkb > 0) ? __ldg(sa_p) : 0.f;
                    sb_n = (col_ok && nkb > 0) ? __ldg(sb_p) : 0.f;
                }
                next_loaded = false;
            }
            for (int kb = 0; kb < nkb; ++kb) {
                float s = 0.f;
                if (!kGroupK) {
                    s = sa_n * sb_n;
                    if (kb + 1 < nkb) {
                        sa_n = row_ok ? __ldg(sa_p + (int64_t)(kb + 1) * a.M_total) : 0.f;
                        sb_n = col_ok ? __ldg(sb_p + kb + 1) : 0.f;
                    } else if (tile + (int)gridDim.x < total) {
                        // the next tile's first scales
                        const Tile Tn = decode_tile(tile + (int)gridDim.x, s_tiles, s_off, a, nt, e_hint);
                        const float* nsa;
                        const float* nsb;
                        bool nrok, ncok;
                        scale_ptrs(Tn, nsa, nsb, nrok, ncok);
                        sa_n = (nrok && Tn.nkb > 0) ? __ldg(nsa) : 0.f;
                        sb_n = (ncok && Tn.nkb > 0) ? __ldg(nsb) : 0.f;
                        next_loaded = true;
                    }
                }
                if (!mbar_wait(tfull_bar(buf), bphase, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(32 * quarter) << 16) + buf * BN + kCols * grp;
                if (!kGroupK) {
                    const float2 s2 = make_float2(s, s);
#pragma unroll
                    for (int ch = 0; ch < kCols / 64; ++ch) {
                        uint32_t p[64];
                        tmem_ld64(taddr + 64 * ch, p);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            acc[32 * ch + i] = __ffma2_rn(
                                make_float2(__uint_as_float(p[2 * i]), __uint_as_float(p[2 * i + 1])),
                                s2, acc[32 * ch + i]);
                    }
                } else {
                    // Both scales vary along the tile here (row scale of A, column
                    // scale of B), so the partial is read in the 16x256b shape: a
                    // thread holds 4 rows x 32 columns (rows g4 + 8k, columns
                    // 8j + c2 + {0,1} of each 64-column group) and needs only 16
                    // column-scale pairs and 4 row scales per K block, read from the
                    // producer's slot with distinct addresses instead of 128
                    // broadcast values.  acc[(cg * 8 + j) * 4 + k] holds row k's pair.
                    const float* slot = reinterpret_cast<const float*>(
                        smem + kOffScales + (sc % kScaleSlots) * kScaleSlotBytes);
                    ++sc;
                    float sak[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) sak[k] = slot[32 * quarter + g4 + 8 * k];
                    const float* sbp = slot + BM + kCols * grp + c2;
#pragma unroll
                    for (int cg = 0; cg < 2; ++cg) {
                        float2 sb2[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            sb2[j] = col_ok ? *reinterpret_cast<const float2*>(sbp + 64 * cg + 8 * j)
                                            : make_float2(0.f, 0.f);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t p[32];
                            tmem_ld16x256_x8(taddr + ((16u * h) << 16) + 64 * cg, p);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
#pragma unroll
                                for (int kk = 0; kk < 2; ++kk) {
                                    const int k = 2 * h + kk;
                                    const float2 w = __fmul2_rn(sb2[j], make_float2(sak[k], sak[k]));
                                    acc[(cg * 8 + j) * 4 + k] = __ffma2_rn(
                                        make_float2(__uint_as_float(p[4 * j + 2 * kk]),
                                                    __uint_as_float(p[4 * j + 2 * kk + 1])),
                                        w, acc[(cg * 8 + j) * 4 + k]);
                                }
                            }
                        }
                    }
                }
                // gate/up mode: the last K block's buffer carries the up values to
                // the gate warps in the epilogue and is released there
                if (kGroupK || !kSwiglu || kb + 1 < nkb) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty_bar(buf));
                }
                buf ^= 1u;
                if (buf == 0) bphase ^= 1u;
            }
            if (!ok) break;
            if (!kGroupK && kSwiglu) {
                // Epilogue (gate/up): h = silu(gate) * up for this row's 128
                // columns, quantized as one 1x128 tile, the work split evenly:
                // the gate warps form h for columns 0..63, the up warps for
                // 64..127.  Each warpgroup parks the half of its accumulators
                // the other needs in its own (already read) part of the last K
                // block's TMEM buffer -- gate columns 64..127 at 64..127, up
                // columns 0..63 at 128..191, same lanes -- and reads the other
                // half back; the two row maxima meet through shared memory.
                const uint32_t lbuf = buf ^ 1u;
                const uint32_t lb = tmem_base + ((uint32_t)(32 * quarter) << 16) + lbuf * BN;
                const uint32_t xp = (xphase >> lbuf) & 1u;
                xphase ^= 1u << lbuf;
                if (grp == 0)
                    tmem_st64(lb + 64, acc + 32);
                else
                    tmem_st64(lb + 128, acc);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(xchg_bar(lbuf, grp));
                if (!mbar_wait(xchg_bar(lbuf, grp ^ 1), xp, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float amax = 0.f;
                // my 64 columns' h into acc[0..31]
                if (grp == 0) {
                    uint32_t u[64];
                    tmem_ld64(lb + 128, u);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        acc[i].x = silu_mul(acc[i].x, __uint_as_float(u[2 * i]));
                        acc[i].y = silu_mul(acc[i].y, __uint_as_float(u[2 * i + 1]));
                        amax = fmaxf(amax, fmaxf(fabsf(acc[i].x), fabsf(acc[i].y)));
                    }
                } else {
                    uint32_t g[64];
                    tmem_ld64(lb + 64, g);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        acc[i].x = silu_mul(__uint_as_float(g[2 * i]), acc[32 + i].x);
                        acc[i].y = silu_mul(__uint_as_float(g[2 * i + 1]), acc[32 + i].y);
                        amax = fmaxf(amax, fmaxf(fabsf(acc[i].x), fabsf(acc[i].y)));
                    }
                }
                float* s_amax = reinterpret_cast<float*>(smem + kOffScales) + (2 * lbuf) * BM;
                s_amax[grp * BM + r] = amax;
                __syncwarp();
                if (lane == 0) mbar_arrive(amax_bar(lbuf, grp));
                if (!mbar_wait(amax_bar(lbuf, grp ^ 1), xp, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                amax = fmaxf(amax, s_amax[(grp ^ 1) * BM + r]);
                const float sc = fg8::tile_scale(amax);
                const fg8::QScale q = fg8::make_qscale(sc);
                // 64 codes of this thread's row through the warp's staging rows:
                // each store writes 8 rows x 64 bytes
                uint32_t* stg = reinterpret_cast<uint32_t*>(smem + kOffStage) + ep * 32 * kStageWords;
                uint4* my_row = reinterpret_cast<uint4*>(stg + lane * kStageWords);
                const int sub = ((lane >> 2) & 1) * 4 + (lane >> 3);
                const int quad = lane & 3;
                const int I = a.N / 2;
                uint8_t* ob = static_cast<uint8_t*>(a.out) + col0 + 64 * grp + 16 * quad;
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
                    uint2 c[2];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int base = 8 * w4 + 4 * hh;   // float2 index: 8 values
                        c[hh] = fg8::quant8f(acc[base], acc[base + 1], acc[base + 2], acc[base + 3], q);
                    }
                    my_row[w4] = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
                }
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int rr = 8 * g + sub;
                    const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStageWords + 4 * quad);
                    if (32 * quarter + rr < rows_valid)
                        *reinterpret_cast<uint4*>(ob + (int64_t)(out_row0 + 32 * quarter + rr) * I) = v;
                }
                __syncwarp();
                if (grp == 0 && row_ok) a.out_scale[(int64_t)(col0 / 128) * a.M_total + out_row0 + r] = sc;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(lbuf));
            } else if (kGroupK) {
                // Epilogue (contraction-grouped, fp32, full 128-row tiles): each
                // warp writes its 32 rows x 128 columns as four 32 x 32 boxes,
                // two at a time through its two 4 KB staging buffers, and
                // TMA-stores them; the stores drain while the warp moves on.
                // The output is written once and never read here, so its lines
                // go first when L2 needs room.
                // 128-byte swizzle: 16-byte chunk c of box row rr sits at chunk
                // c ^ (rr & 7); the four lanes of a row write 32 contiguous bytes,
                // so each 8-byte store of the warp is two conflict-free wavefronts.
                if (col_ok) {
#pragma unroll
                    for (int pr = 0; pr < 2; ++pr) {
                        if (lane == 0 && nbox > 0) bulk_wait_read<0>();   // both buffers drained
                        __syncwarp();
                        uint8_t* stg = smem + kOffStage + ep * kTmaStagePerWarp;
#pragma unroll
                        for (int bb = 0; bb < 2; ++bb) {
                            const int bx = 2 * pr + bb;   // box: columns 32 bx .. of the half
                            uint8_t* box = stg + bb * kBoxBytes;
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int j = 4 * (bx & 1) + jj;
                                const int chunk = 2 * jj + ((lane & 3) >> 1);
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int rr = g4 + 8 * k;
                                    *reinterpret_cast<float2*>(box + rr * 128 + ((chunk ^ (rr & 7)) << 4) +
                                                               8 * (lane & 1)) = acc[(pr * 8 + j) * 4 + k];
                                }
                            }
                        }
                        fence_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            const uint64_t stream_out = l2_policy_evict_first();
#pragma unroll
                            for (int bb = 0; bb < 2; ++bb)
                                tma_store_2d_hint(&tmOut, smem_u32(stg + bb * kBoxBytes), col0 + 64 * pr + 32 * bb,
                                                  out_row0 + 32 * quarter, stream_out);
                            bulk_commit();
                        }
                        ++nbox;
                    }
                }
            } else if (kCombine && col_ok) {
                // Epilogue (combine): every row times its gate weight, added
                // into its token's row of the fp32 output with 16-byte
                // reductions; staged like the fp32 epilogue so that each
                // reduction instruction covers 8 rows x 64 contiguous bytes
                uint32_t* stg = reinterpret_cast<uint32_t*>(smem + kOffStage) + ep * 32 * kStageWords;
                uint4* my_row = reinterpret_cast<uint4*>(stg + lane * kStageWords);
                const int sub = ((lane >> 2) & 1) * 4 + (lane >> 3);
                const int quad = lane & 3;
                const bool mine_ok = 32 * quarter + lane < rows_valid;
                const int my_tok = mine_ok ? a.row_tok[out_row0 + 32 * quarter + lane] : -1;
                const float my_w = mine_ok ? a.row_w[out_row0 + 32 * quarter + lane] : 0.f;
                float* ob = static_cast<float*>(a.out) + col0 + 4 * quad;
#pragma unroll
                for (int ch = 0; ch < kCols / 16; ++ch) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        my_row[q] = make_uint4(__float_as_uint(acc[8 * ch + 2 * q].x),
                                               __float_as_uint(acc[8 * ch + 2 * q].y),
                                               __float_as_uint(acc[8 * ch + 2 * q + 1].x),
                                               __float_as_uint(acc[8 * ch + 2 * q + 1].y));
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int rr = 8 * g + sub;
                        const int t = __shfl_sync(0xFFFFFFFFu, my_tok, rr);
                        const float wgt = __shfl_sync(0xFFFFFFFFu, my_w, rr);
                        const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStageWords + 4 * quad);
                        if (t >= 0)
                            red_add_v4(ob + (int64_t)t * a.N + 16 * ch, wgt * __uint_as_float(v.x),
                                       wgt * __uint_as_float(v.y), wgt * __uint_as_float(v.z),
                                       wgt * __uint_as_float(v.w));
                    }
                    __syncwarp();
                }
            } else if (col_ok) {
            // Epilogue: 16 words of each row at a time go through this warp's
            // staging rows, then every store instruction writes 8 rows x 64
            // contiguous bytes (whole sectors) instead of 32 scattered pieces.
                uint32_t* stg = reinterpret_cast<uint32_t*>(smem + kOffStage) + ep * 32 * kStageWords;
                uint4* my_row = reinterpret_cast<uint4*>(stg + lane * kStageWords);
                const int sub = ((lane >> 2) & 1) * 4 + (lane >> 3);  // rows g*8+sub, conflict-free
                const int quad = lane & 3;
                if (a.out_f32) {
                    float* ob = static_cast<float*>(a.out) + col0 + 4 * quad;
#pragma unroll
                    for (int ch = 0; ch < kCols / 16; ++ch) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            my_row[q] = make_uint4(__float_as_uint(acc[8 * ch + 2 * q].x),
                                                   __float_as_uint(acc[8 * ch + 2 * q].y),
                                                   __float_as_uint(acc[8 * ch + 2 * q + 1].x),
                                                   __float_as_uint(acc[8 * ch + 2 * q + 1].y));
                        __syncwarp();
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int rr = 8 * g + sub;
                            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStageWords + 4 * quad);
                            if (32 * quarter + rr < rows_valid)
                                *reinterpret_cast<uint4*>(ob + (int64_t)(out_row0 + 32 * quarter + rr) * a.N + 16 * ch) = v;
                        }
                        __syncwarp();
                    }
                } else {
                    uint16_t* ob = static_cast<uint16_t*>(a.out) + col0 + 8 * quad;
#pragma unroll
                    for (int ch = 0; ch < kCols / 32; ++ch) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            my_row[q] = make_uint4(pack_bf16x2(acc[16 * ch + 4 * q + 0].x, acc[16 * ch + 4 * q + 0].y),
                                                   pack_bf16x2(acc[16 * ch + 4 * q + 1].x, acc[16 * ch + 4 * q + 1].y),
                                                   pack_bf16x2(acc[16 * ch + 4 * q + 2].x, acc[16 * ch + 4 * q + 2].y),
                                                   pack_bf16x2(acc[16 * ch + 4 * q + 3].x, acc[16 * ch + 4 * q + 3].y));
                        __syncwarp();
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int rr = 8 * g + sub;
                            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * kStageWords + 4 * quad);
                            if (32 * quarter + rr < rows_valid)
                                *reinterpret_cast<uint4*>(ob + (int64_t)(out_row0 + 32 * quarter + rr) * a.N + 32 * ch) = v;
                        }
                        __syncwarp();
                    }
                }
            }
        }
        // TMA stores read shared memory asynchronously: let them finish
        if (kGroupK && lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (kGroupK && warp == 2 && lane == 0 && !*abort_flag) {
        // Each producer took tickets until one was past the last tile, so after
        // a clean launch the counter ends at tiles + CTAs.  The last CTA to get
        // here checks it: another launch sharing the workspace leaves a
        // different count.
        __threadfence();
        if (atomicAdd(a.ws + 1, 1u) == gridDim.x - 1) {
            __threadfence();
            const unsigned tiles = (unsigned)a.E * (unsigned)(a.M_total / BM) * (unsigned)((a.N + BN - 1) / BN);
            if (*reinterpret_cast<volatile unsigned*>(a.ws) != tiles + gridDim.x)
                fg8::set_status(a.status, FG8_ERR_WORKSPACE_SHARED);
        }
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// Combine mode: each routed row's token and gate weight, as
// fg8_unpermute_combine forms them (the token's kept affinities summed in
// fp32 in slot order, one IEEE division); rows outside [0, offsets[E]) get
// token -1.
__global__ void combine_row_weights(const int32_t* __restrict__ offsets, int E, int64_t M_total,
                                    const int32_t* __restrict__ row_token,
                                    const int32_t* __restrict__ token_row,
                                    const float* __restrict__ affinity, int64_t T, int k, int normalize,
                                    int32_t* __restrict__ row_tok, float* __restrict__ row_w) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= M_total) return;
    const int64_t R = offsets[E];
    int32_t t = -1;
    float w = 0.f;
    if (r < R) {
        const int32_t tt = row_token[r];
        if (tt >= 0 && tt < T) {
            const int32_t* tr = token_row + (int64_t)tt * k;
            const float* af = affinity + (int64_t)tt * k;
            float sum = 0.f, mine = 0.f;
            bool found = false;
            for (int j = 0; j < k; ++j) {
                const int32_t rj = tr[j];
                if (rj < 0 || rj >= R) continue;
                sum = __fadd_rn(sum, af[j]);
                if (rj == r) {
                    mine = af[j];
                    found = true;
                }
            }
            if (found) {
                t = tt;
                w = !normalize ? mine : (sum == 0.f ? 0.f : __fdiv_rn(mine, sum));
            }
        }
    }
    row_tok[r] = t;
    row_w[r] = w;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// 2-D u8 matrix [rows][cols], box rows x 128 bytes, 128-byte swizzle (operand tiles).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return fg8h::make_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, 128,
                                    box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

extern "C" size_t fg8_grouped_gemm_workspace(int group_mode) {
    return group_mode == FG8_GROUP_K ? kGroupKWorkspace : 0;
}

extern "C" fg8_status fg8_grouped_gemm(const uint8_t* a, const float* sa, const uint8_t* b,
                                       const float* sb, const int32_t* offsets, int64_t M_total,
                                       int N, int K, int E, int group_mode, int bscale_mode,
                                       int out_dtype, void* out, void* workspace, size_t ws_bytes,
                                       int32_t* dev_status, fg8_stream_t stream) {
    if (!a || !sa || !b || !sb || !offsets || !out) return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128 || M_total < 0)
        return FG8_ERR_INVALID_ARG;
    if (E > kMaxE) return FG8_ERR_UNSUPPORTED;
    if (out_dtype != FG8_OUT_BF16 && out_dtype != FG8_OUT_F32) return FG8_ERR_INVALID_ARG;
    if (!fg8h::aligned16(a) || !fg8h::aligned16(b) || !fg8h::aligned16(out) ||
        !fg8h::aligned16(sb) || (reinterpret_cast<uintptr_t>(sa) & 3) ||
        (reinterpret_cast<uintptr_t>(offsets) & 3))
        return FG8_ERR_INVALID_ARG;
    if (M_total > INT32_MAX) return FG8_ERR_UNSUPPORTED;

    const int64_t nt = (N + BN - 1) / BN;
    int64_t max_tiles;
    CUtensorMap mA, mB, mOut;
    if (group_mode == FG8_GROUP_M) {
        if (bscale_mode != FG8_BSCALE_BLOCK128) return FG8_ERR_UNSUPPORTED;
        if (M_total == 0) return FG8_OK;
        if ((int64_t)E * N > INT32_MAX) return FG8_ERR_UNSUPPORTED;
        max_tiles = (M_total / BM + E) * nt;
        if (!make_map(&mA, a, (uint64_t)M_total, (uint64_t)K, BM) ||
            !make_map(&mB, b, (uint64_t)E * N, (uint64_t)K, BN))
            return FG8_ERR_CUDA;
        mOut = mA;   // unused by the row-grouped epilogue
    } else if (group_mode == FG8_GROUP_K) {
        if (bscale_mode != FG8_BSCALE_ROW128) return FG8_ERR_UNSUPPORTED;
        if (M_total % 128 || !fg8h::aligned16(sa)) return FG8_ERR_INVALID_ARG;
        if (!workspace || !fg8h::aligned16(workspace) || ws_bytes < kGroupKWorkspace)
            return FG8_ERR_INVALID_ARG;
        if (out_dtype != FG8_OUT_F32) return FG8_ERR_UNSUPPORTED;
        if (M_total == 0) return FG8_OK;
        if ((int64_t)E * M_total > INT32_MAX) return FG8_ERR_UNSUPPORTED;
        max_tiles = (int64_t)E * (M_total / BM) * nt;
        if (!make_map(&mA, a, (uint64_t)M_total, (uint64_t)K, BM) ||
            !make_map(&mB, b, (uint64_t)N, (uint64_t)K, BN) ||
            !fg8h::make_tensor_map_2d(&mOut, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, out,
                                      (uint64_t)E * M_total, (uint64_t)N, 32, 32,
                                      CU_TENSOR_MAP_SWIZZLE_128B))
            return FG8_ERR_CUDA;
    } else {
        return FG8_ERR_INVALID_ARG;
    }
    if (max_tiles > INT32_MAX) return FG8_ERR_UNSUPPORTED;

    auto kern = group_mode == FG8_GROUP_K ? grouped_gemm_kernel<true> : grouped_gemm_kernel<false>;
    const uint32_t smem_bytes =
        group_mode == FG8_GROUP_K ? Layout<true>::kSmemBytes : Layout<false>::kSmemBytes;
    // the warpgroup register split must fit in what the CTA is launched with
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, (const void*)kern) != cudaSuccess) return FG8_ERR_CUDA;
    const int launch_regs = group_mode == FG8_GROUP_K ? Warps<true>::kLaunchRegs : Warps<false>::kLaunchRegs;
    const int threads = group_mode == FG8_GROUP_K ? Warps<true>::kThreads : Warps<false>::kThreads;
    if (fa.numRegs < launch_regs) return FG8_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes) !=
        cudaSuccess)
        return FG8_ERR_CUDA;
    GemmArgs args;
    args.sa = sa;
    args.sb = sb;
    args.offsets = offsets;
    args.M_total = M_total;
    args.N = N;
    args.K = K;
    args.E = E;
    args.mode = group_mode;
    args.out_f32 = out_dtype == FG8_OUT_F32;
    args.out = out;
    args.status = dev_status;
    args.ws = nullptr;
    args.swiglu = 0;
    args.out_scale = nullptr;
    args.row_tok = nullptr;
    args.row_w = nullptr;
    if (group_mode == FG8_GROUP_K) {
        args.ws = static_cast<unsigned int*>(workspace);
        if (cudaMemsetAsync(workspace, 0, kGroupKWorkspace, (cudaStream_t)stream) != cudaSuccess)
            return FG8_ERR_CUDA;
    }
    int64_t grid = fg8h::num_sms();
    if (grid > max_tiles) grid = max_tiles;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, threads, smem_bytes, (cudaStream_t)stream>>>(mA, mB, mOut, args);
    return fg8h::launch_status();
}

extern "C" fg8_status fg8_grouped_gemm_swiglu_quant(const uint8_t* a, const float* sa,
                                                    const uint8_t* b, const float* sb,
                                                    const int32_t* offsets, int64_t M_total, int I,
                                                    int K, int E, uint8_t* hq, float* sh,
                                                    int32_t* dev_status, fg8_stream_t stream) {
    if (!a || !sa || !b || !sb || !offsets || !hq || !sh) return FG8_ERR_INVALID_ARG;
    if (E < 1 || I < 128 || K < 128 || I % 128 || K % 128 || M_total < 0)
        return FG8_ERR_INVALID_ARG;
    if (E > kMaxE) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(a) || !fg8h::aligned16(b) || !fg8h::aligned16(hq) ||
        (reinterpret_cast<uintptr_t>(sa) & 3) || (reinterpret_cast<uintptr_t>(sb) & 3) ||
        (reinterpret_cast<uintptr_t>(sh) & 3) || (reinterpret_cast<uintptr_t>(offsets) & 3))
        return FG8_ERR_INVALID_ARG;
    if (M_total > INT32_MAX || (int64_t)E * 2 * I > INT32_MAX) return FG8_ERR_UNSUPPORTED;
    if (M_total == 0) return FG8_OK;
    const int64_t max_tiles = (M_total / BM + E) * (int64_t)(I / 128);
    if (max_tiles > INT32_MAX) return FG8_ERR_UNSUPPORTED;
    CUtensorMap mA, mB;
    // B boxes of 128 rows: a tile's gate block and up block land as the two
    // halves of the 256-row operand tile
    if (!make_map(&mA, a, (uint64_t)M_total, (uint64_t)K, BM) ||
        !make_map(&mB, b, (uint64_t)E * 2 * I, (uint64_t)K, 128))
        return FG8_ERR_CUDA;
    auto kern = grouped_gemm_kernel<false, true>;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, (const void*)kern) != cudaSuccess) return FG8_ERR_CUDA;
    if (fa.numRegs < Warps<false>::kLaunchRegs) return FG8_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout<false>::kSmemBytes) != cudaSuccess)
        return FG8_ERR_CUDA;
    GemmArgs args;
    args.sa = sa;
    args.sb = sb;
    args.offsets = offsets;
    args.M_total = M_total;
    args.N = 2 * I;
    args.K = K;
    args.E = E;
    args.mode = FG8_GROUP_M;
    args.out_f32 = 0;
    args.out = hq;
    args.status = dev_status;
    args.ws = nullptr;
    args.swiglu = 1;
    args.out_scale = sh;
    args.row_tok = nullptr;
    args.row_w = nullptr;
    int64_t grid = fg8h::num_sms();
    if (grid > max_tiles) grid = max_tiles;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, Warps<false>::kThreads, Layout<false>::kSmemBytes, (cudaStream_t)stream>>>(
        mA, mB, mA, args);
    return fg8h::launch_status();
}

extern "C" size_t fg8_grouped_gemm_combine_workspace(int64_t M_total) {
    return M_total > 0 ? (size_t)M_total * 8 : 0;
}

extern "C" fg8_status fg8_grouped_gemm_combine(const uint8_t* a, const float* sa, const uint8_t* b,
                                               const float* sb, const int32_t* offsets,
                                               int64_t M_total, int N, int K, int E,
                                               const int32_t* row_token, const int32_t* token_row,
                                               const float* affinity, int64_t T, int k,
                                               int normalize, float* out, void* workspace,
                                               size_t ws_bytes, int32_t* dev_status,
                                               fg8_stream_t stream) {
    if (!a || !sa || !b || !sb || !offsets || !row_token || !token_row || !affinity || !out)
        return FG8_ERR_INVALID_ARG;
    if (E < 1 || N < 128 || K < 128 || N % 128 || K % 128 || M_total < 0 || T < 0)
        return FG8_ERR_INVALID_ARG;
    if (k < 1 || k > 16) return FG8_ERR_INVALID_ARG;
    if (E > kMaxE) return FG8_ERR_UNSUPPORTED;
    if (!fg8h::aligned16(a) || !fg8h::aligned16(b) || !fg8h::aligned16(out) || !fg8h::aligned16(sb) ||
        (reinterpret_cast<uintptr_t>(sa) & 3) || (reinterpret_cast<uintptr_t>(offsets) & 3) ||
        (reinterpret_cast<uintptr_t>(row_token) & 3) || (reinterpret_cast<uintptr_t>(token_row) & 3) ||
        (reinterpret_cast<uintptr_t>(affinity) & 3))
        return FG8_ERR_INVALID_ARG;
    if (M_total > INT32_MAX || T > INT32_MAX || (int64_t)E * N > INT32_MAX || T * k > INT32_MAX)
        return FG8_ERR_UNSUPPORTED;
    if (M_total > 0 && T > 0 &&
        (!workspace || !fg8h::aligned16(workspace) || ws_bytes < fg8_grouped_gemm_combine_workspace(M_total)))
        return FG8_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (T > 0 && cudaMemsetAsync(out, 0, (size_t)T * N * sizeof(float), st) != cudaSuccess)
        return FG8_ERR_CUDA;
    if (M_total == 0 || T == 0) return FG8_OK;
    int32_t* row_tok = static_cast<int32_t*>(workspace);
    float* row_w = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + (size_t)M_total * 4);
    combine_row_weights<<<(unsigned)((M_total + 255) / 256), 256, 0, st>>>(
        offsets, E, M_total, row_token, token_row, affinity, T, k, normalize, row_tok, row_w);
    if (cudaGetLastError() != cudaSuccess) return FG8_ERR_CUDA;
    const int64_t nt = N / BN + (N % BN != 0);
    const int64_t max_tiles = (M_total / BM + E) * nt;
    if (max_tiles > INT32_MAX) return FG8_ERR_UNSUPPORTED;
    CUtensorMap mA, mB;
    if (!make_map(&mA, a, (uint64_t)M_total, (uint64_t)K, BM) ||
        !make_map(&mB, b, (uint64_t)E * N, (uint64_t)K, BN))
        return FG8_ERR_CUDA;
    auto kern = grouped_gemm_kernel<false, false, true>;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, (const void*)kern) != cudaSuccess) return FG8_ERR_CUDA;
    if (fa.numRegs < Warps<false>::kLaunchRegs) return FG8_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout<false>::kSmemBytes) != cudaSuccess)
        return FG8_ERR_CUDA;
    GemmArgs args;
    args.sa = sa;
    args.sb = sb;
    args.offsets = offsets;
    args.M_total = M_total;
    args.N = N;
    args.K = K;
    args.E = E;
    args.mode = FG8_GROUP_M;
    args.out_f32 = 1;
    args.out = out;
    args.status = dev_status;
    args.ws = nullptr;
    args.swiglu = 0;
    args.out_scale = nullptr;
    args.row_tok = row_tok;
    args.row_w = row_w;
    int64_t grid = fg8h::num_sms();
    if (grid > max_tiles) grid = max_tiles;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, Warps<false>::kThreads, Layout<false>::kSmemBytes, st>>>(mA, mB, mA, args);
    return fg8h::launch_status();
}
