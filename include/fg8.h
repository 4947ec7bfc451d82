/*
 * fg8.h -- C ABI of libfg8: FP8 fine-grained quantization for MoE expert
 * layers on NVIDIA B200 (sm_100a).
 *
 * The operations follow two pages:
 *  [K2] "Kakao Kanana-2 pre-training deep dive" (devday.kr), the FP8 paragraph:
 *       fine-grained FP8 scaling with 1x128 activation tiles and 128x128
 *       weight blocks; one MoE quantization kernel for all experts instead of
 *       one expert after another; a kernel that transposes block-quantized
 *       weights for backward, so only the forward FP8 weight is stored.
 *  [DS] "DeepSeek-V3 summary" (theinnovators.zone), sec. 2.1 (sigmoid
 *       affinity, top-K routing, per-expert bias, no token dropping) and
 *       sec. 2.2 "FP8 mixed precision training" (most GEMMs in FP8, 1x128 /
 *       128x128 tile/block quantization, high-precision accumulation).
 *
 * Numerics (one reading of the pages, which fix neither format nor formula):
 * FP8 is OCP E4M3FN.  For each tile or block with largest magnitude amax,
 *     s = fp32(amax / 448)   (s = 1 when amax == 0),
 *     q = E4M3(fp32(x / s))  round to nearest, ties to even, saturating at
 *                            +-448, sign of zero kept.
 * s is the dequantization multiplier: x ~= q * s.  NaN/Inf inputs are outside
 * the contract (their outputs are unspecified).
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, never synchronizes the stream and keeps no state
 *    between calls, so calls on different streams with disjoint buffers
 *    (workspaces included) are independent.  One stated exception: the
 *    allocation-free quantizer's scratch (fg8_quantize_act_noalloc) is device
 *    memory of the library.  `stream` is a cudaStream_t (NULL = the legacy
 *    stream).
 *  - bf16 data is passed as uint16_t bit patterns.  FP8 data as uint8_t.
 *  - Calls are asynchronous.  Argument errors are found on the host and
 *    returned immediately (nothing is launched).  Launch failures return
 *    FG8_ERR_CUDA.  Conditions only the device can see (an expert id out of
 *    range, a bounded wait that ran out) are written to *dev_status (a device
 *    int32 that the caller zeroes once and reads after synchronizing); the
 *    library sets it to the first such fg8_status and never clears it.
 *    Kernels never trap.
 *  - Buffers that TMA reads (the GEMM operands) and every FP8/bf16 buffer
 *    must be 16-byte aligned; row strides are implied by the sizes.
 */
#ifndef FG8_H
#define FG8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FG8_OK = 0,
    FG8_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment   */
    FG8_ERR_UNSUPPORTED = 2,   /* valid but not implemented combination  */
    FG8_ERR_CUDA = 3,          /* a CUDA runtime/launch error            */
    FG8_ERR_BAD_EXPERT_ID = 4, /* device: an id outside [0, E) was met   */
    FG8_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out         */
    FG8_ERR_WORKSPACE_SHARED = 6 /* device: a workspace was in use by an
                                    overlapping call (results invalid)   */
} fg8_status;

typedef enum { FG8_ROWWISE = 1, FG8_COLWISE = 2 } fg8_act_layout;
typedef enum { FG8_OUT_BF16 = 0, FG8_OUT_F32 = 1 } fg8_out_dtype;
typedef enum { FG8_GROUP_M = 0, FG8_GROUP_K = 1 } fg8_group_mode;
typedef enum { FG8_BSCALE_BLOCK128 = 0, FG8_BSCALE_ROW128 = 1 } fg8_bscale_mode;

typedef void* fg8_stream_t; /* cudaStream_t */

/*
 * fg8_quantize_act -- 1x128 activation quantization to E4M3 with one fp32
 * scale per tile, fused with the token-to-expert permute, all experts in one
 * launch ([K2] FP8 paragraph; [DS] sec. 2.1 no token dropping, sec. 2.2
 * 1x128 tiles).
 *
 * layout = FG8_ROWWISE, topk_ids != NULL  (forward dispatch):
 *   x          bf16  [T][K], K % 128 == 0
 *   topk_ids   int32 [T][k], expert ids in [0, E)
 *   xq         E4M3  [R][K], R = T*k; rows grouped by expert, experts in
 *              ascending order, inside an expert by ascending (token, slot)
 *   sa         fp32  [K/128][R]: sa[kb*R + r] is the scale of row r, K block kb
 *   row_token  int32 [R]:   token of each row
 *   token_row  int32 [T*k]: row of each (token, slot); -1 for a bad id
 *   offsets_out int32 [E+1]: expert e owns rows [offsets_out[e], offsets_out[e+1])
 *   workspace  >= fg8_quantize_act_workspace(T, k, E) bytes, 16-byte aligned
 *   Each token row is read once and its codes written to its k rows.  An id
 *   outside [0, E) sets *dev_status = FG8_ERR_BAD_EXPERT_ID; that pair gets
 *   no row (the tail rows of xq/sa/row_token stay unwritten).
 *   This mode uses a cooperative launch (all CTAs resident) with grid-wide
 *   barriers whose waits are bounded (FG8_ERR_TIMEOUT in *dev_status).
 *   Calls that share one workspace must not overlap on the GPU.
 *
 * layout = FG8_ROWWISE, topk_ids == NULL  (rows already in expert order):
 *   x [T][K] -> xq [T][K], sa [K/128][T]; k must be 1; E, offsets and index
 *   maps are ignored (may be 0/NULL); workspace may be NULL.
 *
 * layout = FG8_COLWISE  (weight-gradient operands: 1x128 along the token axis)
 *   Logical rows r in [0, R), R = T*k, are grouped by expert through
 *   offsets_in [E+1] (device, offsets_in[E] == R).  If row_token != NULL it
 *   is an INPUT [R] and logical row r is x[row_token[r]] (x has T rows);
 *   otherwise k must be 1 and logical row r is x[r].  Each expert's rows are
 *   cut into tiles of 128 consecutive rows, the last one zero-padded; every
 *   (column, tile) gets one scale (padding takes no part in amax, and is
 *   written as code 0x00).  With P = fg8_colwise_capacity(R, E):
 *   xqT        E4M3 [K][P]: token axis contiguous; expert e occupies columns
 *              [offsets_out[e], offsets_out[e+1]) of each row
 *   saT        fp32 [P/128][K]: saT[(p/128)*K + c]
 *   offsets_out int32 [E+1]: padded offsets, sum of ceil(T_e/128)*128
 *   Columns past offsets_out[E] are not written.  xq, sa, token_row and
 *   workspace are unused.
 */
fg8_status fg8_quantize_act(const uint16_t* x, int64_t T, int64_t K,
                            const int32_t* topk_ids, int k, int E,
                            const int32_t* offsets_in, int layout,
                            uint8_t* xq, float* sa,
                            int32_t* row_token, int32_t* token_row, int32_t* offsets_out,
                            uint8_t* xqT, float* saT,
                            void* workspace, size_t ws_bytes,
                            int32_t* dev_status, fg8_stream_t stream);

/*
 * fg8_route_quantize_act -- routing fused in front of the permuting
 * quantizer: the sigmoid-affinity top-K choice of fg8_route_topk ([DS] sec.
 * 2.1) and the 1x128 permute + quantize of fg8_quantize_act ([K2] FP8
 * paragraph; [DS] sec. 2.2) in one cooperative launch.  The routing phase
 * histograms the experts it picks as it goes, so the ids are never read
 * back for counting.  Outputs are exactly those of fg8_route_topk followed
 * by fg8_quantize_act (permuting mode) on its ids.
 *   logits fp32 [T][E], bias fp32 [E]      as for fg8_route_topk
 *   x bf16 [T][K], K % 128 == 0            as for fg8_quantize_act
 *   topk_ids int32 [T][k], affinity fp32 [T][k]   outputs (as fg8_route_topk)
 *   xq, sa, row_token, token_row, offsets_out, workspace, ws_bytes
 *                                          as for fg8_quantize_act
 *   1 <= k <= min(16, E), E <= 1024.  NaN logits are outside the contract.
 *   T == 0 only zeroes offsets_out.  The grid-wide barriers' waits are
 *   bounded (FG8_ERR_TIMEOUT in *dev_status).
 */
fg8_status fg8_route_quantize_act(const float* logits, const float* bias,
                                  const uint16_t* x, int64_t T, int64_t K, int k, int E,
                                  int32_t* topk_ids, float* affinity,
                                  uint8_t* xq, float* sa, int32_t* row_token,
                                  int32_t* token_row, int32_t* offsets_out,
                                  void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, fg8_stream_t stream);

/*
 * fg8_quantize_act_noalloc -- the permuting mode of fg8_quantize_act
 * (layout FG8_ROWWISE with topk_ids) for callers that cannot allocate device
 * memory, such as a plugin whose host framework owns every allocation and
 * passes only inputs and outputs, or a path that must never enter the
 * allocator.  The pages have no counterpart of this call; it exists for
 * those callers only.
 *   Arguments and outputs are those of fg8_quantize_act in the permuting
 *   mode, without the workspace.  The scratch the kernel needs is a ~1 MiB
 *   array inside libfg8 itself (a __device__ variable, so every GPU that
 *   loads the library holds it until the process exits); the call allocates
 *   nothing and calls no allocating routine.
 *   Limit: E <= 256; a larger E returns FG8_ERR_UNSUPPORTED.
 *   The first call on each device (with that device current) looks up the
 *   array's device address and keeps it for that device's context; the first
 *   call after the context is replaced (cudaDeviceReset, or the primary
 *   context released and created again) looks it up again.  Make those calls
 *   before any stream capture.  All calls on a device share the array: calls
 *   that overlap on the GPU race with each other.  The library resets what
 *   must start at zero on every call.
 */
fg8_status fg8_quantize_act_noalloc(const uint16_t* x, int64_t T, int64_t K,
                                    const int32_t* topk_ids, int k, int E,
                                    uint8_t* xq, float* sa, int32_t* row_token,
                                    int32_t* token_row, int32_t* offsets_out,
                                    int32_t* dev_status, fg8_stream_t stream);

/* Workspace bytes needed by fg8_quantize_act in the permuting mode. */
size_t fg8_quantize_act_workspace(int64_t T, int k, int E);

/* Width P of the column-wise buffers for R logical rows over E experts:
 * round_up(R + 127*E, 128). */
int64_t fg8_colwise_capacity(int64_t R, int E);

/*
 * fg8_quantize_weight -- 128x128 block quantization of the weights of all
 * experts in one launch ([K2] FP8 paragraph; [DS] sec. 2.2 128x128 blocks).
 *   w   bf16 [E][N][K], N % 128 == 0, K % 128 == 0, 16-byte aligned
 *   wq  E4M3 [E][N][K], 16-byte aligned
 *   sw  fp32 [E][N/128][K/128]
 *   dev_status  optional (NULL allowed) device int32: a block whose load
 *       never arrives (bounded wait) gets a NaN scale and FG8_ERR_TIMEOUT
 *       is recorded here.
 */
fg8_status fg8_quantize_weight(const uint16_t* w, int E, int N, int K,
                               uint8_t* wq, float* sw, int32_t* dev_status,
                               fg8_stream_t stream);

/*
 * fg8_quantize_weight_transposed -- fg8_quantize_weight that also writes the
 * block-transposed copy the backward pass needs (the output of
 * fg8_transpose_blockq) from the codes it has just formed, so producing both
 * costs one read of w instead of an extra read of wq.  Outputs are identical
 * to fg8_quantize_weight followed by fg8_transpose_blockq.
 *   w, wq, sw, dev_status  as for fg8_quantize_weight
 *   wqT  E4M3 [E][K][N], 16-byte aligned
 *   swT  fp32 [E][K/128][N/128]
 */
fg8_status fg8_quantize_weight_transposed(const uint16_t* w, int E, int N, int K,
                                          uint8_t* wq, float* sw, uint8_t* wqT, float* swT,
                                          int32_t* dev_status, fg8_stream_t stream);

/*
 * fg8_transpose_blockq -- transpose an already block-quantized weight and its
 * scale grid for backward, so only the forward FP8 copy is stored ([K2] FP8
 * paragraph, last sentence).  Pure byte/scale moves: because the blocks are
 * square, dequant(transpose(Q)) == transpose(dequant(Q)) exactly.
 *   wq  E4M3 [E][N][K] -> wqT E4M3 [E][K][N]
 *   sw  fp32 [E][N/128][K/128] -> swT fp32 [E][K/128][N/128]
 */
fg8_status fg8_transpose_blockq(const uint8_t* wq, const float* sw, int E, int N, int K,
                                uint8_t* wqT, float* swT, fg8_stream_t stream);

/*
 * fg8_grouped_gemm -- grouped FP8 GEMM with fine-grained scales: at every
 * 128-wide K step the tensor-core partial product is promoted into an fp32
 * accumulator with the activation tile scale and the weight block scale
 * ([DS] sec. 2.2 most GEMMs in FP8, high-precision accumulation; [K2] FP8
 * paragraph).  Runs on tcgen05 tensor cores (TMEM accumulators, TMA loads).
 * out[r][n] = sum_kb sA(r,kb) * sB(n,kb) * sum_{k in kb} A[r][k] * B[n][k].
 *
 * group_mode = FG8_GROUP_M (forward / dgrad; variable rows per expert):
 *   a        E4M3 [M_total][K]; sa fp32 [K/128][M_total]
 *   b        E4M3 [E][N][K] (K-major, e.g. fg8_quantize_weight's wq, or
 *            fg8_transpose_blockq's wqT for dgrad)
 *   sb       fp32 [E][N/128][K/128] (bscale_mode = FG8_BSCALE_BLOCK128)
 *   offsets  int32 [E+1] on the device: expert e owns rows
 *            [offsets[e], offsets[e+1]); offsets[E] <= M_total
 *   out      [M_total][N] bf16 or fp32; rows outside [0, offsets[E]) are
 *            not written.  An expert with no rows costs nothing.
 *   N % 128 == 0, K % 128 == 0, E <= 1024.  workspace may be NULL.
 *
 * group_mode = FG8_GROUP_K (weight gradient; variable contraction per expert):
 *   a        E4M3 [M_total][K], sa fp32 [K/128][M_total]
 *   b        E4M3 [N][K],       sb fp32 [K/128][N] (bscale_mode = FG8_BSCALE_ROW128)
 *   offsets  int32 [E+1] on the device, multiples of 128, offsets[E] <= K
 *            (fg8_quantize_act COLWISE's offsets_out; K = its capacity P)
 *   out      [E][M_total][N]: out[e] = sum over columns [offsets[e],
 *            offsets[e+1]) of the contraction; an expert with no columns gets
 *            zeros.  M_total % 128 == 0, N % 128 == 0, K % 128 == 0, E <= 1024;
 *            sa and sb 16-byte aligned (the scale vectors are bulk-copied);
 *            out_dtype must be FG8_OUT_F32 (weight gradients are accumulated
 *            in fp32; other dtypes return FG8_ERR_UNSUPPORTED).
 *   The tiles are handed out at run time from a counter in `workspace`
 *   (>= fg8_grouped_gemm_workspace(FG8_GROUP_K) bytes, 16-byte aligned,
 *   zeroed by the call on `stream` before the launch).  Calls that share a
 *   workspace must not overlap on the GPU; when they do, the tiles of a
 *   launch are no longer processed exactly once, and the last CTA of the
 *   launch reports FG8_ERR_WORKSPACE_SHARED in *dev_status (the output is
 *   then invalid).
 *
 * The fp32 output is the accumulator; the bf16 output is its round-to-
 * nearest-even conversion.  dev_status may be NULL only if no device-side
 * condition needs reporting is acceptable to the caller (bounded waits still
 * end the kernel).
 */
fg8_status fg8_grouped_gemm(const uint8_t* a, const float* sa,
                            const uint8_t* b, const float* sb,
                            const int32_t* offsets, int64_t M_total, int N, int K, int E,
                            int group_mode, int bscale_mode, int out_dtype, void* out,
                            void* workspace, size_t ws_bytes,
                            int32_t* dev_status, fg8_stream_t stream);

/* Workspace bytes fg8_grouped_gemm needs in `group_mode` (0 for FG8_GROUP_M). */
size_t fg8_grouped_gemm_workspace(int group_mode);

/*
 * fg8_grouped_gemm_swiglu_quant -- the expert up-projection with its gated
 * activation and the down-projection's 1x128 input quantization fused into
 * the GEMM epilogue.  The pages combine FP8 GEMMs with separately written
 * non-GEMM kernels ([K2] FP8 paragraph; [DS] sec. 2.2, FP8 mixed precision)
 * and quantize every activation that enters an FP8 GEMM in 1x128 tiles; they
 * do not name the expert's activation function.  Reading taken here: the
 * gated SiLU of DeepSeek-style experts,
 *   h[r][i] = silu(G[r][i]) * U[r][i],  silu(g) = g / (1 + exp(-g)),
 * with G and U the fp32 accumulators of the row-grouped GEMM against the gate
 * and up halves of b (promoted exactly as in fg8_grouped_gemm), and h
 * quantized from fp32 (never rounded to bf16) as 1x128 tiles: for every row
 * r and block c, sh[c][r] = amax/448 (1 for an all-zero tile) and
 * hq[r][128c + j] = E4M3 RNE-satfinite(h / sh[c][r]).
 *   a        E4M3 [M_total][K]; sa fp32 [K/128][M_total]
 *   b        E4M3 [E][2I][K]: rows [0, I) of expert e are the gate weight,
 *            rows [I, 2I) the up weight (fg8_quantize_weight of [E][2I][K])
 *   sb       fp32 [E][2I/128][K/128]
 *   offsets  int32 [E+1] on the device, as for FG8_GROUP_M
 *   hq       E4M3 [M_total][I] and sh fp32 [I/128][M_total] (the layout
 *            fg8_grouped_gemm takes as a and sa); rows outside
 *            [0, offsets[E]) are not written
 *   I % 128 == 0, K % 128 == 0, E <= 1024; a, b, hq 16-byte aligned.
 * silu uses the fast exponential and division intrinsics (a few ulp in fp32).
 * Errors as fg8_grouped_gemm; a timed-out internal wait writes
 * FG8_ERR_TIMEOUT to *dev_status.
 */
fg8_status fg8_grouped_gemm_swiglu_quant(const uint8_t* a, const float* sa,
                                         const uint8_t* b, const float* sb,
                                         const int32_t* offsets, int64_t M_total, int I, int K,
                                         int E, uint8_t* hq, float* sh, int32_t* dev_status,
                                         fg8_stream_t stream);

/*
 * fg8_route_topk -- sigmoid-affinity top-K routing with a per-expert bias
 * ([DS] sec. 2.1: sigmoid affinity scores, top-K experts per token, a
 * per-expert bias term adjusted for load balance instead of an auxiliary
 * loss).  Reading taken here: the bias enters only the choice, the gate
 * values use the plain affinities.  For every token t and expert e, in fp32:
 *   s[e] = 1 / (1 + exp(-logits[t][e]))   (IEEE add and divide, accurate exp)
 *   c[e] = s[e] + bias[e]
 * ids[t][0..k) are the k experts with the largest c, in descending c, ties
 * to the lower expert index; affinity[t][j] = s[ids[t][j]].  The outputs feed
 * fg8_quantize_act (ids) and fg8_unpermute_combine (affinity).
 *   logits fp32 [T][E]; bias fp32 [E]; ids int32 [T][k]; affinity fp32 [T][k]
 *   1 <= k <= min(16, E), E <= 1024.  NaN logits are outside the contract.
 *   A bias of -inf masks an expert: it ranks after every finite score and,
 *   if fewer than k experts are finite, masked experts fill the remaining
 *   slots in ascending index order (so every row still holds k valid ids).
 */
fg8_status fg8_route_topk(const float* logits, const float* bias, int64_t T, int E, int k,
                          int32_t* ids, float* affinity, fg8_stream_t stream);

/*
 * fg8_unpermute_combine -- the layer output of routed tokens: every token's
 * expert output rows (one per routed slot, in the permuted expert order that
 * fg8_quantize_act produced) summed with the gate weights ([DS] sec. 2.1:
 * sigmoid affinity scores, top-K experts per token, no token dropping).  The
 * page does not spell out how the affinities of the chosen experts become
 * weights; reading taken here: they are normalized to sum 1 over the token's
 * kept slots (normalize = 1), or used as given (normalize = 0).
 *   out[t][c] = sum_{j < k, slot kept} w[t][j] * y[token_row[t*k + j]][c]
 *   w[t][j]   = normalize ? affinity[t][j] / (sum of the kept affinity[t][.])
 *                         : affinity[t][j]
 * A slot is kept when token_row[t*k + j] is in [0, R); others (-1 = no row)
 * add nothing.  Arithmetic in fp32 with every operation rounded to nearest
 * (the affinity sum and the weighted sum in slot order j = 0, 1, ...); a
 * normalized token whose kept affinities sum to 0 gets zeros.
 *   y          bf16 [R][C] (e.g. the down-projection output), R may be 0
 *   token_row  int32 [T*k] (fg8_quantize_act's token_row)
 *   affinity   fp32 [T][k]
 *   out        [T][C], bf16 (RNE of the fp32 sum) or fp32 (out_dtype)
 *   1 <= k <= 16, C % 8 == 0; y and out 16-byte aligned.
 */
fg8_status fg8_unpermute_combine(const uint16_t* y, int64_t R, int C, const int32_t* token_row,
                                 const float* affinity, int64_t T, int k, int normalize,
                                 int out_dtype, void* out, fg8_stream_t stream);

/*
 * fg8_grouped_gemm_combine -- the down-projection and the combine in one
 * launch: the row-grouped FP8 GEMM of fg8_grouped_gemm (FG8_GROUP_M,
 * FG8_BSCALE_BLOCK128, the same promotion), whose epilogue multiplies every
 * routed row by its gate weight and adds it into its token's row of the fp32
 * output, instead of writing the rows for a separate fg8_unpermute_combine
 * ([DS] sec. 2.1: the layer output is the affinity-weighted sum of the
 * token's expert outputs).
 *   out[t][c] = sum_{j < k, slot kept} w[t][j] * Y[token_row[t*k + j]][c]
 * with Y the fp32 GEMM result (not rounded to bf16) and w[t][j] exactly as in
 * fg8_unpermute_combine (kept affinities summed in fp32 in slot order, one
 * IEEE division when normalize = 1).  Each product w * Y is rounded to fp32
 * and added with an fp32 reduction in L2; the order of a token's k additions
 * is not specified (it can differ between runs, within fp32 rounding).
 *   a, sa, b, sb, offsets, M_total, N, K, E: as fg8_grouped_gemm, FG8_GROUP_M
 *   row_token  int32 [M_total] (fg8_quantize_act's row_token)
 *   token_row  int32 [T*k]; affinity fp32 [T][k]; 1 <= k <= 16
 *   out        fp32 [T][N], zeroed by the call on the stream, then summed into
 *   workspace  >= fg8_grouped_gemm_combine_workspace(M_total) bytes, 16-byte
 *              aligned, caller-owned: every row's token and weight; calls that
 *              overlap on the GPU need their own
 * Rows with no kept slot (or outside [0, offsets[E])) add nothing; tokens
 * with no rows get zeros.  Errors as fg8_grouped_gemm.
 */
size_t fg8_grouped_gemm_combine_workspace(int64_t M_total);
fg8_status fg8_grouped_gemm_combine(const uint8_t* a, const float* sa, const uint8_t* b,
                                    const float* sb, const int32_t* offsets, int64_t M_total,
                                    int N, int K, int E, const int32_t* row_token,
                                    const int32_t* token_row, const float* affinity, int64_t T,
                                    int k, int normalize, float* out, void* workspace,
                                    size_t ws_bytes, int32_t* dev_status, fg8_stream_t stream);

/*
 * Expert-parallel exchange of FP8 rows (the data plane around an all-to-all;
 * [DS] sec. 2.2: training on a cluster of NVLink / InfiniBand nodes with FP8
 * communication, and the experts spread over the GPUs).  With W ranks, rank
 * r owns the E_loc = E / W experts [r E_loc, (r + 1) E_loc).  After
 * fg8_quantize_act the rows bound for rank r are the contiguous range
 * [offsets_out[r E_loc], offsets_out[(r + 1) E_loc]) of xq, so the codes are
 * sent as they are; these calls prepare the scales for the trip, merge what
 * arrives into local expert order, and send expert outputs back.  The
 * exchange itself (e.g. NCCL all-to-all) is the caller's.
 *
 * fg8_ep_pack_scales -- sa fp32 [K/128][R] (fg8_quantize_act's layout) ->
 *   sa_rows fp32 [R][K/128], so the rows of each destination carry their
 *   scales as one contiguous range too.  K % 128 == 0.
 */
fg8_status fg8_ep_pack_scales(const float* sa, int64_t R, int64_t K, float* sa_rows,
                              fg8_stream_t stream);

/*
 * fg8_ep_unpack -- on the receiving rank: the W incoming segments, source 0
 * first, each holding its rows grouped by local expert in ascending order,
 * become the local expert order (expert-major, then source rank, then the
 * source's own order), ready for fg8_grouped_gemm (GROUP_M).
 *   recv_xq      E4M3 [R_recv][K] and recv_sa fp32 [R_recv][K/128]: received
 *   counts       int32 [W][E_loc] on the device: rows source s sent for local
 *                expert e (their sum must be R_recv)
 *   xq, sa       E4M3 [R_recv][K], fp32 [K/128][R_recv]: local rows
 *   offsets      int32 [E_loc + 1]: local expert e owns rows
 *                [offsets[e], offsets[e + 1])
 *   recv_to_local int32 [R_recv]: local row of each received row (the
 *                combine's fg8_gather_rows map)
 *   W * E_loc <= 2048; K % 128 == 0; xq and recv_xq 16-byte aligned.  If the
 *   counts do not sum to R_recv, nothing is written and *dev_status gets
 *   FG8_ERR_INVALID_ARG.
 */
fg8_status fg8_ep_unpack(const uint8_t* recv_xq, const float* recv_sa, const int32_t* counts,
                         int W, int E_loc, int64_t R_recv, int64_t K, uint8_t* xq, float* sa,
                         int32_t* offsets, int32_t* recv_to_local, int32_t* dev_status,
                         fg8_stream_t stream);

/*
 * fg8_gather_rows -- out[i] = in[map[i]] for n rows of row_bytes bytes (a
 * multiple of 16; in and out 16-byte aligned).  The combine side of the
 * exchange: with map = recv_to_local, the expert outputs return to the order
 * in which their rows arrived, so after the reverse all-to-all each rank
 * holds its rows in its own permuted order (fg8_unpermute_combine's input).
 * A map entry outside [0, n_in) leaves its output row untouched and writes
 * FG8_ERR_INVALID_ARG to *dev_status.
 */
fg8_status fg8_gather_rows(const void* in, int64_t n_in, int64_t row_bytes, const int32_t* map,
                           int64_t n, void* out, int32_t* dev_status, fg8_stream_t stream);

/*
 * fg8_selftest_wait_timeout -- diagnostic of the failure-detection path (the
 * pages have no counterpart).  Runs one of the library's bounded device waits
 * on a condition that nothing satisfies, so that it runs out after its limit
 * (about 2 s), writes FG8_ERR_TIMEOUT to *dev_status and returns; the context
 * stays usable.  Faults nothing.
 *   which = 0: the grid-wide barrier of the permuting quantizer
 *              (scratch: one device uint32, cleared by the call)
 *   which = 1: the mbarrier wait used by the GEMM pipeline (scratch unused)
 */
fg8_status fg8_selftest_wait_timeout(int which, uint32_t* scratch, int32_t* dev_status,
                                     fg8_stream_t stream);

/* Static string naming a status. */
const char* fg8_status_string(fg8_status s);

#ifdef __cplusplus
}
#endif

#endif /* FG8_H */
