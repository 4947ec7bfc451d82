/*
 * fg8_oracle.c -- CPU oracle for the FP8 fine-grained MoE quantization path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain definition that the
 * CUDA library is checked against.  It shares no code, header, table or
 * constant generator with the CUDA path, and only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  Nothing in the
 * product calls it; the product has no CPU fallback.
 *
 * What it computes, and where that comes from:
 *
 *  - Granularity.  Activations are quantized in 1x128 tiles (one scale per row
 *    and 128 consecutive K elements), weights in 128x128 blocks (one scale per
 *    block): Kanana-2 pre-training deep dive (devday.kr), FP8 paragraph, and
 *    the DeepSeek-V3 summary (theinnovators.zone), sec. 2.2 "FP8 mixed
 *    precision training", second bullet.
 *  - One pass over all experts; a transpose of the block-quantized weight (and
 *    its scale grid) for backward, so only the forward FP8 weight is stored:
 *    Kanana-2 deep dive, FP8 paragraph, last two sentences.
 *  - Every (token, slot) is dispatched (no token dropping), so the permuted
 *    activation has exactly T*k rows: DeepSeek-V3 summary, sec. 2.1, routing
 *    bullets.
 *  - GEMM partial sums are promoted to high precision (fp32 on the GPU); the
 *    oracle sums in fp64: DeepSeek-V3 summary, sec. 2.2, third bullet.
 *  - Around the expert GEMMs (each with the reading it takes stated where it
 *    is defined below): sigmoid-affinity top-K routing with a per-expert bias
 *    and the weighted combine of a token's expert outputs (DeepSeek-V3
 *    summary, sec. 2.1), and the gated activation between the two expert
 *    GEMMs, re-quantized in 1x128 tiles for the second (Kanana-2 deep dive,
 *    FP8 paragraph; DeepSeek-V3 summary, sec. 2.2).  These are computed in
 *    fp64 throughout.
 *
 * The pages fix neither the FP8 format nor the scale formula.  This oracle
 * takes one reading and states it: OCP "E4M3FN" (bias 7, no infinities, NaN =
 * S.1111.111, largest finite 448, subnormal step 2^-9); per tile
 *     amax = max |x|                         (exact, in fp32)
 *     s    = fp32_RN(amax / 448)             (s = 1 when amax == 0)
 *     q_i  = E4M3_RNE_satfinite(fp32_RN(x_i / s))
 * where E4M3 rounding is to the nearest representable value, ties to the
 * code with an even last bit, and any magnitude >= 448 maps to 448 (sign
 * kept, -0 -> 0x80).  Inputs are bf16; NaN/Inf inputs are outside the
 * contract.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no fast-math, so
 * float '/' is IEEE division rounded to nearest even and subnormals are kept).
 */

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E4M3FN from its definition                                               */
/* ------------------------------------------------------------------------ */

/* Exact value of an E4M3FN code: sign bit 7, exponent bits 6..3 (bias 7),
 * mantissa bits 2..0.  Exponent field 0 is subnormal: M * 2^-9.  The pattern
 * S.1111.111 is NaN; every other code is finite. */
double fg8o_e4m3_decode(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* magnitudes of codes 0x00..0x7E, ascending (the encoding is monotonic) */
static double g_mag[127];
static int g_mag_ready = 0;

static void init_mag(void)
{
    if (g_mag_ready)
        return;
    for (int c = 0; c < 127; ++c)
        g_mag[c] = fg8o_e4m3_decode((uint8_t)c);
    g_mag_ready = 1;
}

/* Round a finite fp32 value to E4M3FN: nearest representable magnitude,
 * ties to the even code, saturating at 448.  The comparison is exact: the
 * midpoint of two adjacent E4M3 values has at most 5 significant bits, so it
 * is exact in double, and so is the fp32 input. */
uint8_t fg8o_e4m3_encode(float v)
{
    init_mag();
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v))
        return (uint8_t)(0x7F | sign);
    double a = fabs((double)v);
    if (a >= 448.0)
        return (uint8_t)(0x7E | sign);
    /* largest code c with g_mag[c] <= a (binary search over the table) */
    int lo = 0, hi = 126;          /* g_mag[lo] <= a < g_mag[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (g_mag[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    double midpoint = 0.5 * (g_mag[lo] + g_mag[hi]);
    int pick;
    if (a < midpoint)
        pick = lo;
    else if (a > midpoint)
        pick = hi;
    else
        pick = (lo & 1) ? hi : lo;     /* tie: the code whose last bit is 0 */
    return (uint8_t)(pick | sign);
}

void fg8o_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = fg8o_e4m3_encode(v[i]);
}

float fg8o_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* scale of a tile whose largest magnitude is amax */
float fg8o_tile_scale(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return amax / 448.0f;                      /* one IEEE fp32 division */
}

static uint8_t quant_elem(float x, float s)
{
    float q = x / s;                            /* fp32_RN(x / s) */
    return fg8o_e4m3_encode(q);
}

/* ------------------------------------------------------------------------ */
/* token -> expert permutation                                              */
/* ------------------------------------------------------------------------ */

/* counts[e] = #{(t,j): ids[t*k+j] == e}; offsets = exclusive prefix sum
 * (offsets[E] = number of valid pairs); rows of expert e are filled in
 * ascending t, then ascending j.  row_token[row] = t, token_row[t*k+j] = row.
 * A pair whose id is outside [0,E) gets no row (token_row = -1).  Returns the
 * number of such pairs. */
int64_t fg8o_route(const int32_t* ids, int64_t T, int k, int E,
                   int32_t* counts, int32_t* offsets,
                   int32_t* row_token, int32_t* token_row)
{
    int64_t bad = 0;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t p = 0; p < T * k; ++p) {
        int32_t e = ids[p];
        if (e < 0 || e >= E)
            ++bad;
        else
            ++counts[e];
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int e = 0; e < E; ++e)
        fill[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int32_t e = ids[t * k + j];
            if (e < 0 || e >= E) {
                token_row[t * k + j] = -1;
                continue;
            }
            int32_t row = fill[e]++;
            row_token[row] = (int32_t)t;
            token_row[t * k + j] = row;
        }
    }
    free(fill);
    return bad;
}

/* ------------------------------------------------------------------------ */
/* 1x128 activation quantization, fused with the permute                    */
/* ------------------------------------------------------------------------ */

/* Quantize one 1x128 tile of bf16 values (contiguous). */
static void quant_row_tile(const uint16_t* x, uint8_t* q, float* scale)
{
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
        float a = fabsf(fg8o_bf16_to_f32(x[i]));
        if (a > amax)
            amax = a;
    }
    float s = fg8o_tile_scale(amax);
    for (int i = 0; i < 128; ++i)
        q[i] = quant_elem(fg8o_bf16_to_f32(x[i]), s);
    *scale = s;
}

/* Row-wise activation quantization.
 *   x      bf16 [T][K] (row-major), K % 128 == 0
 *   ids    int32 [T][k] expert ids, or NULL: identity (rows already in order,
 *          R = T, no index maps are written)
 *   xq     E4M3 [R][K], R = T*k (rows in expert order)
 *   sa     fp32 [K/128][R]: sa[kb*R + r] is the scale of row r, K block kb
 *   row_token, token_row, offsets: as fg8o_route (ignored when ids == NULL)
 * Returns the number of out-of-range ids. */
int64_t fg8o_quantize_act_rowwise(const uint16_t* x, int64_t T, int64_t K,
                                  const int32_t* ids, int k, int E,
                                  uint8_t* xq, float* sa,
                                  int32_t* row_token, int32_t* token_row,
                                  int32_t* offsets)
{
    int64_t KB = K / 128;
    if (ids == NULL) {
        int64_t R = T;
        for (int64_t r = 0; r < R; ++r)
            for (int64_t kb = 0; kb < KB; ++kb)
                quant_row_tile(x + r * K + kb * 128, xq + r * K + kb * 128, &sa[kb * R + r]);
        return 0;
    }
    int64_t R = T * k;
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int64_t bad = fg8o_route(ids, T, k, E, counts, offsets, row_token, token_row);
    free(counts);
    /* destination row r holds token row_token[r]; quantize it there */
    for (int64_t r = 0; r < offsets[E]; ++r) {
        int64_t t = row_token[r];
        for (int64_t kb = 0; kb < KB; ++kb)
            quant_row_tile(x + t * K + kb * 128, xq + r * K + kb * 128, &sa[kb * R + r]);
    }
    return bad;
}

/* Column-wise (token-axis) 1x128 quantization per expert, for the weight
 * gradient.  Logical row r (0 <= r < offsets[E]) is src[row_map[r]] when
 * row_map != NULL, else src[r]; src is bf16 [*][C].  Expert e owns logical
 * rows [offsets[e], offsets[e+1]); they are cut into tiles of 128 consecutive
 * rows, the last one padded with zeros.  Each (column c, tile) has one scale;
 * the padding takes no part in amax and is written as 0x00.
 *   padoff  int32 [E+1]: padoff[e] = sum over e' < e of ceil(T_e'/128)*128
 *   xqT     E4M3 [C][P_cap]: xqT[c*P_cap + padoff[e] + i] = code of row
 *           offsets[e] + i, column c (token axis contiguous)
 *   sT      fp32 [P_cap/128][C]: sT[(padoff[e]/128 + b)*C + c]
 */
void fg8o_quantize_act_colwise(const uint16_t* src, int64_t C, const int32_t* row_map,
                               const int32_t* offsets, int E, int64_t P_cap,
                               uint8_t* xqT, float* sT, int32_t* padoff)
{
    padoff[0] = 0;
    for (int e = 0; e < E; ++e) {
        int64_t Te = offsets[e + 1] - offsets[e];
        padoff[e + 1] = padoff[e] + (int32_t)(((Te + 127) / 128) * 128);
    }
    for (int e = 0; e < E; ++e) {
        int64_t Te = offsets[e + 1] - offsets[e];
        int64_t ntile = (Te + 127) / 128;
        for (int64_t b = 0; b < ntile; ++b) {
            int64_t n_in = Te - b * 128 < 128 ? Te - b * 128 : 128;
            for (int64_t c = 0; c < C; ++c) {
                float amax = 0.0f;
                for (int64_t i = 0; i < n_in; ++i) {
                    int64_t r = offsets[e] + b * 128 + i;
                    int64_t sr = row_map ? row_map[r] : r;
                    float a = fabsf(fg8o_bf16_to_f32(src[sr * C + c]));
                    if (a > amax)
                        amax = a;
                }
                float s = fg8o_tile_scale(amax);
                sT[(padoff[e] / 128 + b) * C + c] = s;
                for (int64_t i = 0; i < 128; ++i) {
                    uint8_t q = 0x00;
                    if (i < n_in) {
                        int64_t r = offsets[e] + b * 128 + i;
                        int64_t sr = row_map ? row_map[r] : r;
                        q = quant_elem(fg8o_bf16_to_f32(src[sr * C + c]), s);
                    }
                    xqT[c * P_cap + padoff[e] + b * 128 + i] = q;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* 128x128 weight block quantization, all experts                           */
/* ------------------------------------------------------------------------ */

/* w bf16 [E][N][K]; wq E4M3 [E][N][K]; sw fp32 [E][N/128][K/128]. */
void fg8o_quantize_weight(const uint16_t* w, int64_t E, int64_t N, int64_t K,
                          uint8_t* wq, float* sw)
{
    int64_t NB = N / 128, KB = K / 128;
    for (int64_t e = 0; e < E; ++e)
        for (int64_t nb = 0; nb < NB; ++nb)
            for (int64_t kb = 0; kb < KB; ++kb) {
                const uint16_t* blk = w + (e * N + nb * 128) * K + kb * 128;
                uint8_t* qblk = wq + (e * N + nb * 128) * K + kb * 128;
                float amax = 0.0f;
                for (int i = 0; i < 128; ++i)
                    for (int j = 0; j < 128; ++j) {
                        float a = fabsf(fg8o_bf16_to_f32(blk[i * K + j]));
                        if (a > amax)
                            amax = a;
                    }
                float s = fg8o_tile_scale(amax);
                for (int i = 0; i < 128; ++i)
                    for (int j = 0; j < 128; ++j)
                        qblk[i * K + j] = quant_elem(fg8o_bf16_to_f32(blk[i * K + j]), s);
                sw[(e * NB + nb) * KB + kb] = s;
            }
}

/* ------------------------------------------------------------------------ */
/* transpose of a block-quantized weight and its scale grid                 */
/* ------------------------------------------------------------------------ */

/* wqT[e][k][n] = wq[e][n][k]; swT[e][kb][nb] = sw[e][nb][kb]. */
void fg8o_transpose_blockq(const uint8_t* wq, const float* sw, int64_t E, int64_t N,
                           int64_t K, uint8_t* wqT, float* swT)
{
    int64_t NB = N / 128, KB = K / 128;
    for (int64_t e = 0; e < E; ++e) {
        for (int64_t n = 0; n < N; ++n)
            for (int64_t kk = 0; kk < K; ++kk)
                wqT[(e * K + kk) * N + n] = wq[(e * N + n) * K + kk];
        for (int64_t nb = 0; nb < NB; ++nb)
            for (int64_t kb = 0; kb < KB; ++kb)
                swT[(e * KB + kb) * NB + nb] = sw[(e * NB + nb) * KB + kb];
    }
}

/* ------------------------------------------------------------------------ */
/* GEMM references in fp64                                                  */
/* ------------------------------------------------------------------------ */

static double g_dq[256];
static int g_dq_ready = 0;

static void init_dq(void)
{
    if (g_dq_ready)
        return;
    for (int c = 0; c < 256; ++c)
        g_dq[c] = fg8o_e4m3_decode((uint8_t)c);
    g_dq_ready = 1;
}

/* Row-grouped (forward / dgrad) product, one entry at a time:
 *   Y[r][n] = sum_k dq(a[r][k]) * sa[k/128][r] * dq(b[e][n][k]) * sb[e][n/128][k/128]
 * for r in expert e's row range [offsets[e], offsets[e+1]).
 *   a  E4M3 [M_total][K]; sa fp32 [K/128][M_total]
 *   b  E4M3 [E][N][K];    sb fp32 [E][N/128][K/128]
 * For each requested (rows[i], cols[i]): ref[i] = the sum in fp64 and
 * bound[i] = the sum of the absolute values of its terms.  Each term is
 * (dq(a) dq(b)) * (sa sb): the first factor is exact, so is the second
 * (two 24-bit significands), and their product is rounded once in fp64. */
void fg8o_gemm_mgrouped_entries(const uint8_t* a, const float* sa, int64_t M_total,
                                const uint8_t* b, const float* sb,
                                const int32_t* offsets, int E, int64_t N, int64_t K,
                                const int64_t* rows, const int64_t* cols, int64_t n_entries,
                                double* ref, double* bound)
{
    init_dq();
    int64_t NB = N / 128, KB = K / 128;
    for (int64_t i = 0; i < n_entries; ++i) {
        int64_t r = rows[i], n = cols[i];
        int e = 0;
        while (e < E && !(offsets[e] <= r && r < offsets[e + 1]))
            ++e;
        double acc = 0.0, abs_acc = 0.0;
        if (e < E) {
            for (int64_t kk = 0; kk < K; ++kk) {
                int64_t kb = kk / 128;
                double scale = (double)sa[kb * M_total + r] * (double)sb[(e * NB + n / 128) * KB + kb];
                double prod = g_dq[a[r * K + kk]] * g_dq[b[(e * N + n) * K + kk]];
                double term = prod * scale;
                acc += term;
                abs_acc += fabs(term);
            }
        }
        ref[i] = acc;
        bound[i] = abs_acc;
    }
}

/* ------------------------------------------------------------------------ */
/* gated activation of the up-projection, re-quantized in 1x128 tiles        */
/* ------------------------------------------------------------------------ */

/* The pages run most GEMMs in FP8 and quantize every activation that enters
 * one in 1x128 tiles (Kanana-2 deep dive, FP8 paragraph; DeepSeek-V3 summary,
 * sec. 2.2); they do not name the experts' activation.  Reading taken: the
 * gated SiLU of DeepSeek-style experts,
 *     h = silu(g) * u,   silu(g) = g / (1 + exp(-g)),
 * evaluated in fp64 from the fp64 up-projection (g: gate half, u: up half),
 * then rounded once to fp32 and quantized as 1x128 tiles exactly as above
 * (amax of the fp32 values, s = fp32_RN(amax / 448), q = E4M3(fp32_RN(h / s))).
 *   G, U  fp64 [R][I] (row-major), I % 128 == 0
 *   h     fp64 [R][I] out: the activation before rounding (may be NULL)
 *   hq    E4M3 [R][I];  sh fp32 [I/128][R]: sh[c*R + r] scales row r, block c */
void fg8o_swiglu_quantize(const double* G, const double* U, int64_t R, int64_t I,
                          double* h, uint8_t* hq, float* sh)
{
    float* hf = (float*)malloc(sizeof(float) * 128);
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t c = 0; c < I / 128; ++c) {
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                int64_t idx = r * I + c * 128 + i;
                double g = G[idx];
                double v = g / (1.0 + exp(-g)) * U[idx];
                if (h)
                    h[idx] = v;
                hf[i] = (float)v;
                if (fabsf(hf[i]) > amax)
                    amax = fabsf(hf[i]);
            }
            float s = fg8o_tile_scale(amax);
            for (int i = 0; i < 128; ++i)
                hq[r * I + c * 128 + i] = quant_elem(hf[i], s);
            sh[c * R + r] = s;
        }
    }
    free(hf);
}

/* ------------------------------------------------------------------------ */
/* sigmoid-affinity top-K routing with a per-expert bias                    */
/* ------------------------------------------------------------------------ */

/* DeepSeek-V3 summary, sec. 2.1: sigmoid affinity scores, the top-K experts
 * per token, a per-expert bias adjusted for load balance.  Reading taken: the
 * bias only ranks (c = s + b), the affinities written out are s.  In fp64:
 *   s[e] = 1 / (1 + exp(-u[t][e])),  c[e] = s[e] + bias[e]
 * K rounds, each taking the remaining expert with the largest c, ties to the
 * lower index.  ids int32 [T][k]; affinity fp64 [T][k]; score fp64 [T][E]
 * (c of every expert, may be NULL). */
void fg8o_route_topk(const float* logits, const float* bias, int64_t T, int E, int k,
                     int32_t* ids, double* affinity, double* score)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    double* c = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            s[e] = 1.0 / (1.0 + exp(-(double)logits[t * E + e]));
            c[e] = s[e] + (double)bias[e];
            taken[e] = 0;
            if (score)
                score[t * E + e] = c[e];
        }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || c[e] > c[best]))
                    best = e;              /* strict '>' keeps the lower index on ties */
            taken[best] = 1;
            ids[t * k + j] = best;
            affinity[t * k + j] = s[best];
        }
    }
    free(s);
    free(c);
    free(taken);
}

/* ------------------------------------------------------------------------ */
/* unpermute + combine                                                      */
/* ------------------------------------------------------------------------ */

/* Each token's output is the sum of its routed slots' expert rows weighted by
 * the gate values (DeepSeek-V3 summary, sec. 2.1: sigmoid affinities, top-K
 * experts per token).  Reading taken: the gate values are the affinities of
 * the token's kept slots normalized to sum 1 (normalize != 0), or the
 * affinities as given.  A slot is kept when its row is in [0, R).  In fp64:
 *   out[t][c]   = sum_j w[t][j] * y[token_row[t*k + j]][c]
 *   bound[t][c] = sum_j |w[t][j] * y[...][c]|
 *   y bf16 [R][C]; token_row int32 [T*k]; affinity fp32 [T][k]; out, bound fp64 [T][C].
 * A normalized token whose kept affinities sum to 0 gets zeros. */
void fg8o_unpermute_combine(const uint16_t* y, int64_t R, int64_t C, const int32_t* token_row,
                            const float* affinity, int64_t T, int k, int normalize,
                            double* out, double* bound)
{
    for (int64_t t = 0; t < T; ++t) {
        double sum = 0.0;
        for (int j = 0; j < k; ++j) {
            int32_t row = token_row[t * k + j];
            if (row >= 0 && row < R)
                sum += (double)affinity[t * k + j];
        }
        for (int64_t c = 0; c < C; ++c) {
            double acc = 0.0, mag = 0.0;
            for (int j = 0; j < k; ++j) {
                int32_t row = token_row[t * k + j];
                if (row < 0 || row >= R)
                    continue;
                double w = (double)affinity[t * k + j];
                if (normalize)
                    w = sum != 0.0 ? w / sum : 0.0;
                double term = w * (double)fg8o_bf16_to_f32(y[(int64_t)row * C + c]);
                acc += term;
                mag += fabs(term);
            }
            out[t * C + c] = acc;
            bound[t * C + c] = mag;
        }
    }
}

/* Contraction-grouped (weight gradient) product, one entry at a time:
 *   dW[e][m][n] = sum_{p in [padoff[e], padoff[e+1])}
 *                 dq(a[m][p]) * sa[p/128][m] * dq(b[n][p]) * sb[p/128][n]
 *   a  E4M3 [M][P_cap];  sa fp32 [P_cap/128][M]
 *   b  E4M3 [N][P_cap];  sb fp32 [P_cap/128][N]
 * An expert with no tokens has an empty sum: dW = 0. */
void fg8o_gemm_kgrouped_entries(const uint8_t* a, const float* sa, const uint8_t* b,
                                const float* sb, const int32_t* padoff, int E,
                                int64_t M, int64_t N, int64_t P_cap,
                                const int64_t* experts, const int64_t* rows,
                                const int64_t* cols, int64_t n_entries,
                                double* ref, double* bound)
{
    init_dq();
    (void)E;
    for (int64_t i = 0; i < n_entries; ++i) {
        int64_t e = experts[i], m = rows[i], n = cols[i];
        double acc = 0.0, abs_acc = 0.0;
        for (int64_t p = padoff[e]; p < padoff[e + 1]; ++p) {
            int64_t pb = p / 128;
            double scale = (double)sa[pb * M + m] * (double)sb[pb * N + n];
            double prod = g_dq[a[m * P_cap + p]] * g_dq[b[n * P_cap + p]];
            double term = prod * scale;
            acc += term;
            abs_acc += fabs(term);
        }
        ref[i] = acc;
        bound[i] = abs_acc;
    }
}
