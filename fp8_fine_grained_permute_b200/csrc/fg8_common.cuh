// fg8_common.cuh -- device helpers shared by the libfg8 kernels (sm_100a).
//
// The E4M3 quantization step used by every quantize kernel lives here:
//     s = fp32(amax / 448) (1 for an all-zero tile),  q = E4M3_RNE_sat(fp32(x / s))
// following the fine-grained 1x128 / 128x128 scaling of the Kanana-2 deep dive
// (devday.kr, FP8 paragraph) and the DeepSeek-V3 summary (sec. 2.2).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fg8.h"

#define FG8_DEV __device__ __forceinline__

namespace fg8 {

// ---------------------------------------------------------------------------
// status and bounded waits
// ---------------------------------------------------------------------------

// Record the first device-side condition; later ones are dropped.
FG8_DEV void set_status(int32_t* st, int32_t code) {
    if (st != nullptr) atomicCAS(st, 0, code);
}

FG8_DEV uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every spin in this library gives up after this long and reports
// FG8_ERR_TIMEOUT; normal waits last microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// ---------------------------------------------------------------------------
// bf16 unpacking (bit patterns -> fp32, exact)
// ---------------------------------------------------------------------------

FG8_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
FG8_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// E4M3 quantization
// ---------------------------------------------------------------------------

// Scale of a tile with largest magnitude `amax` (IEEE division, no flush).
FG8_DEV float tile_scale(float amax) {
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// Per-tile context of the E4M3 quantization.
//
// The exact code of an element is E4M3(z) with z = fp32(x / s) (IEEE
// division).  Fast path: with r ~ 1/s, E4M3 rounding is monotonic, so if the
// two products x * r(1 - eps) and x * r(1 + eps) get the same code, and the
// interval between them contains z, that shared code is E4M3(z).  r is the
// hardware reciprocal refined by one Newton-Raphson step, r <- r + r (1 - s r),
// so |r - 1/s| <= 2^-23 / s; with the two roundings of the products and the
// rounding of z the interval holds z whenever eps > 5 * 2^-24, and eps = 2^-18
// leaves a factor of ten.  Elements whose two codes differ (a rounding midpoint
// lies inside the interval: about 1 in 8000) and tiles whose scale is
// subnormal (its reciprocal would overflow) take the IEEE division.
struct QScale {
    float s;        // scale (dequantization multiplier)
    float r_lo;     // fp32(r * (1 - 2^-18))
    float r_hi;     // fp32(r * (1 + 2^-18))
    bool exact;     // take the division for every element of the tile
};

FG8_DEV QScale make_qscale(float s) {
    QScale q;
    q.s = s;
    float r0;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r0) : "f"(s));
    const float r = fmaf(r0, fmaf(-s, r0, 1.0f), r0);   // Newton-Raphson step
    q.r_lo = __fmul_rn(r, 1.0f - 0x1p-18f);
    q.r_hi = __fmul_rn(r, 1.0f + 0x1p-18f);
    q.exact = !(s >= 1.17549435e-38f);                   // subnormal scale
    return q;
}

// Two fp32 -> two E4M3 (RNE, saturating to +-448): `lo` in bits 7..0.
FG8_DEV uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

FG8_DEV uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

FG8_DEV uint32_t cvt_e4m3x2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return cvt_e4m3x2(lo, hi);
}

FG8_DEV uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Fast-path codes of 8 bf16 values (one uint4): the codes of x * r(1 - eps)
// and of x * r(1 + eps).  No branch, so callers can keep many of these in
// flight and check them together (exact when lo == hi and !q.exact).
FG8_DEV void quant8_bracket(const uint4& v, const QScale& q, uint2& lo, uint2& hi) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint64_t rl = pack_f32x2(q.r_lo, q.r_lo), rh = pack_f32x2(q.r_hi, q.r_hi);
    uint32_t l[4], h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t x = pack_f32x2(bf16_lo(w[i]), bf16_hi(w[i]));
        l[i] = cvt_e4m3x2(mul_f32x2(x, rl));
        h[i] = cvt_e4m3x2(mul_f32x2(x, rh));
    }
    lo = make_uint2(l[0] | (l[1] << 16), l[2] | (l[3] << 16));
    hi = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

FG8_DEV bool bracket_agrees(const uint2& lo, const uint2& hi) {
    return ((lo.x ^ hi.x) | (lo.y ^ hi.y)) == 0u;
}

// Exact codes of 8 bf16 values by IEEE division (the slow path).
FG8_DEV uint2 quant8_exact(const uint4& v, const QScale& q) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = cvt_e4m3x2(__fdiv_rn(bf16_lo(w[i]), q.s), __fdiv_rn(bf16_hi(w[i]), q.s));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Exact codes of 8 bf16 values for a group whose fast path failed: the
// bracket again, then an IEEE division only for the values whose brackets
// disagree (or all of them for a subnormal scale).  Disagreement is less rare
// than the bracket width suggests: a bf16 value divided by the scale often
// lands exactly on a rounding midpoint between two E4M3 codes (about 5 values
// in a thousand, 4 groups of 8 in a hundred, on normally distributed data).
FG8_DEV uint2 quant8_redo(const uint4& v, const QScale& q) {
    if (q.exact) return quant8_exact(v, q);
    uint2 lo, hi;
    quant8_bracket(v, q, lo, hi);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t& c = j < 4 ? lo.x : lo.y;
        const uint32_t m = 0xFFu << (8 * (j & 3));
        if (((j < 4 ? hi.x : hi.y) ^ c) & m) {
            const float x = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
            c = (c & ~m) | ((cvt_e4m3x2(__fdiv_rn(x, q.s), 0.0f) & 0xFFu) << (8 * (j & 3)));
        }
    }
    return lo;
}

// Warp-cooperative redo of the groups whose fast path failed.  Every lane of
// the warp calls it with its failed groups as bits of `redo` (bit numbers
// < 256); the warp's failed groups are listed in `list` (shared memory, `cap`
// entries) and shared out one per lane, so the warp spends one round on them
// however they fall on its lanes, instead of every lane redoing its own in
// turn.  work(owner_lane, bit) redoes one group.  Returns false, having done
// nothing, when the warp's groups do not fit the list; the caller then redoes
// its own.
template <class F>
FG8_DEV bool coop_redo(uint32_t redo, uint16_t* list, int cap, F work) {
    const int lane = threadIdx.x & 31;
    const uint32_t cnt = __popc(redo);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
    }
    const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (total == 0u) return true;
    if (total > (uint32_t)cap) return false;
    uint32_t pos = incl - cnt;
    while (redo != 0u) {
        const int b = __ffs(redo) - 1;
        redo &= redo - 1u;
        list[pos++] = (uint16_t)((lane << 8) | b);
    }
    __syncwarp();
    for (uint32_t k = lane; k < total; k += 32) {
        const uint32_t e = list[k];
        work((int)(e >> 8), (int)(e & 0xFFu));
    }
    __syncwarp();
    return true;
}

// Quantize 8 bf16 values (one uint4) with scale context q -> 8 codes (uint2).
FG8_DEV uint2 quant8(const uint4& v, const QScale& q) {
    uint2 lo, hi;
    quant8_bracket(v, q, lo, hi);
    if (!q.exact && bracket_agrees(lo, hi)) return lo;
    return quant8_exact(v, q);
}

// Quantize N groups of 8 values sharing one scale context: all fast-path
// codes are formed first (independent work the scheduler can overlap), then
// one combined check decides whether any group needs the exact path.
template <int N>
FG8_DEV void quant8xN(const uint4 (&v)[N], const QScale& q, uint2 (&c)[N]) {
    uint2 hi[N];
    bool ok = !q.exact;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        quant8_bracket(v[i], q, c[i], hi[i]);
        ok &= bracket_agrees(c[i], hi[i]);
    }
    if (!ok) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            if (q.exact || !bracket_agrees(c[i], hi[i])) c[i] = quant8_exact(v[i], q);
    }
}

// Quantize 8 fp32 values (four pairs) with scale context q -> 8 codes.  Same
// bracketed fast path as quant8, on fp32 inputs.
FG8_DEV uint2 quant8f(float2 a, float2 b, float2 c, float2 d, const QScale& q) {
    const float2 v[4] = {a, b, c, d};
    const uint64_t rl = pack_f32x2(q.r_lo, q.r_lo), rh = pack_f32x2(q.r_hi, q.r_hi);
    uint32_t l[4], h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t x = pack_f32x2(v[i].x, v[i].y);
        l[i] = cvt_e4m3x2(mul_f32x2(x, rl));
        h[i] = cvt_e4m3x2(mul_f32x2(x, rh));
    }
    uint2 lo = make_uint2(l[0] | (l[1] << 16), l[2] | (l[3] << 16));
    const uint2 hi = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    if (q.exact || !bracket_agrees(lo, hi)) {
#pragma unroll
        for (int i = 0; i < 4; ++i) l[i] = cvt_e4m3x2(__fdiv_rn(v[i].x, q.s), __fdiv_rn(v[i].y, q.s));
        lo = make_uint2(l[0] | (l[1] << 16), l[2] | (l[3] << 16));
    }
    return lo;
}

// max |x| over 8 bf16 values: magnitudes of non-NaN floats order like their
// bit patterns, so a 16-bit SIMD unsigned max over the sign-cleared words is exact.
FG8_DEV float amax8(const uint4& v) {
    uint32_t m = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    const uint32_t h = max(m & 0xFFFFu, m >> 16);
    return __uint_as_float(h << 16);
}

// ---------------------------------------------------------------------------
// block-wide scan
// ---------------------------------------------------------------------------

// Exclusive scan of s_in[0..n) into s_out[0..n] (s_out[n] = total), n <= 8 * blockDim.
// Must be called by all threads of the block.
FG8_DEV void block_exclusive_scan(const int32_t* s_in, int32_t* s_out, int n,
                               int32_t* s_warp) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5, nw = blockDim.x >> 5;
    const int per = (n + blockDim.x - 1) / blockDim.x;   // <= 8
    int32_t loc[8];
    int32_t sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int idx = t * per + i;
        loc[i] = (i < per && idx < n) ? s_in[idx] : 0;
        sum += loc[i];
    }
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = lane < nw ? s_warp[lane] : 0;
        int32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) s_warp[lane] = wi - w;           // exclusive warp prefix
        if (lane == nw - 1) s_warp[32] = wi;            // block total
    }
    __syncthreads();
    int32_t run = s_warp[warp] + incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int idx = t * per + i;
        if (i < per && idx < n) s_out[idx] = run;
        run += loc[i];
    }
    if (t == 0) s_out[n] = s_warp[32];
    __syncthreads();
}

// ---------------------------------------------------------------------------
// memory helpers
// ---------------------------------------------------------------------------

// streaming 16-byte load (read once; do not keep in L1)
FG8_DEV uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

FG8_DEV uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier on a zero-initialised global counter, for kernels whose
// CTAs are all resident (cooperative launch); `target` = CTAs * phase.
// Returns false (and records FG8_ERR_TIMEOUT) if the wait runs out.
FG8_DEV bool grid_barrier(uint32_t* counter, uint32_t target, int32_t* status) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1u);
        const uint64_t t0 = globaltimer_ns();
        int ok = 1;
        while (ld_acquire_gpu(counter) < target) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                ok = 0;
                set_status(status, FG8_ERR_TIMEOUT);
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

}  // namespace fg8

// Host-side helpers shared by the entry points.
namespace fg8h {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline fg8_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FG8_OK : FG8_ERR_CUDA;
}

int num_sms();  // multiprocessor count of the current device (cached per device)

// 2-D tiled tensor map over a row-major matrix [rows][cols] of `elem_bytes`
// elements (row stride = cols * elem_bytes), box [box_rows][box_cols].
// Returns false if the driver entry point is unavailable or rejects the map.
bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes,
                        const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle);

}  // namespace fg8h
