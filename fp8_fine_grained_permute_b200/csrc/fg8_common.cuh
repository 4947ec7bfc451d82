// fg8_common.cuh -- device helpers shared by the libfg8 kernels (sm_100a).
//
// The E4M3 quantization step used by every quantize kernel lives here:
//     s = fp32(amax / 448) (1 for an all-zero tile),  q = E4M3_RNE_sat(fp32(x / s))
// following the fine-grained 1x128 / 128x128 scaling of the Kanana-2 deep dive
// (devday.kr, FP8 paragraph) and the DeepSeek-V3 summary (sec. 2.2).
#pragma once

#include <cstdint>
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

// Per-tile context for the fast path of fp32(x / s).
//
// The product y' = x * rcp(s) differs from the correctly rounded quotient
// fp32(x / s) by a few fp32 ulps.  E4M3 rounding of a value in the normal
// E4M3 range (|y| >= 2^-6) looks only at the top three fraction bits and
// compares the low 20 fraction bits with the midpoint pattern 0x80000; a
// few-ulp error changes the E4M3 result only if y' lies within those ulps of
// a midpoint.  So: if y' is more than 128 ulps away from every midpoint and
// |y'| >= 2^-6, E4M3(y') == E4M3(fp32(x / s)) exactly; otherwise (and for
// subnormal scales, whose reciprocal overflows) the IEEE division is used.
// The 128-ulp window covers any reciprocal with relative error below 2^-17;
// the hardware approximation is within a few ulps.
struct QScale {
    float s;     // scale (dequantization multiplier)
    float r;     // approximate 1/s
    bool exact;  // take the division for every element
};

FG8_DEV QScale make_qscale(float s) {
    QScale q;
    q.s = s;
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(s));
    q.r = r;
    q.exact = !(s >= 1.17549435e-38f) || !(fabsf(r) <= 3.0e38f);
    return q;
}

// fp32 value whose E4M3 rounding equals that of fp32(x / s).
FG8_DEV float quot(float x, const QScale& q) {
    float y = __fmul_rn(x, q.r);
    uint32_t b = __float_as_uint(y) & 0x7FFFFFFFu;
    uint32_t low = b & 0xFFFFFu;
    bool near_mid = (low - (0x80000u - 128u)) <= 256u;
    bool small = (b < 0x3C800000u) && (b != 0u);      // 0 < |y| < 2^-6
    if (q.exact || near_mid || small) y = __fdiv_rn(x, q.s);
    return y;
}

// Two fp32 -> two E4M3 (RNE, saturating to +-448): `lo` in bits 7..0.
FG8_DEV uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

// Quantize 8 bf16 values (one uint4) with scale context q -> 8 codes (uint2).
FG8_DEV uint2 quant8(const uint4& v, const QScale& q) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = cvt_e4m3x2(quot(bf16_lo(w[i]), q), quot(bf16_hi(w[i]), q));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// max |x| over 8 bf16 values
FG8_DEV float amax8(const uint4& v) {
    float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
    return m;
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

}  // namespace fg8

// Host-side helpers shared by the entry points.
namespace fg8h {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline fg8_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FG8_OK : FG8_ERR_CUDA;
}

int num_sms();  // multiprocessor count of the current device (cached per device)

}  // namespace fg8h
