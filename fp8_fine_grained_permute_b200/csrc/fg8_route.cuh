// fg8_route.cuh -- per-token sigmoid-affinity top-K selection by one warp.
//
// DeepSeek-V3 summary, sec. 2.1: each token's affinity to an expert is a
// sigmoid score, the K experts with the largest scores are chosen, and a
// per-expert bias, adjusted to balance the load, enters the choice (not the
// gate values).  Here s = sigmoid(u) in fp32 (accurate expf, IEEE add and
// divide), the choice ranks c = s + bias with ties to the lower expert index,
// and the affinity handed out for a chosen expert is its s.
//
// Used by the standalone routing kernel (route_topk.cu) and by the routing
// phase of the fused routing + permute + quantize kernel (quant_act.cu).
#pragma once

#include <climits>

#include "fg8_common.cuh"

namespace fg8 {

constexpr int kRouteMaxK = 16;

// (score, index) order of the selection: larger score first, then lower index
FG8_DEV bool route_better(float a, int ia, float b, int ib) { return a > b || (a == b && ia < ib); }

FG8_DEV float route_sigmoid(float u) { return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-u))); }

// One token: u = its E logits, bl = this lane's bias values (experts lane +
// 32 i).  Every lane of the warp calls this; on return lane j < k holds the
// j-th chosen expert (descending c) in `id` and its affinity in `s_out`.
// PER_LANE * 32 >= E.  A bias of -inf masks an expert: it ranks after every
// finite score, and masked experts fill any remaining slots by index.
template <int PER_LANE>
FG8_DEV void route_token(const float* __restrict__ u, const float (&bl)[PER_LANE], int E, int k,
                         int lane, int32_t& id, float& s_out) {
    // only the ranking scores stay in registers; the affinity of a chosen
    // expert is recomputed from its logit by the lane that owns it (same
    // operations, same value)
    float c[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        c[i] = e < E ? __fadd_rn(route_sigmoid(u[e]), bl[i]) : -INFINITY;
    }
    uint32_t taken = 0;   // bit i: expert lane + 32 i already chosen
    id = -1;
    s_out = 0.f;
    for (int j = 0; j < k; ++j) {
        // this lane's best remaining candidate
        float bc = -INFINITY;
        int bi = INT_MAX, bslot = -1;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(taken >> i & 1u) && route_better(c[i], e, bc, bi)) {
                bc = c[i];
                bi = e;
                bslot = i;
            }
        }
        // warp-wide best
        float wc = bc;
        int wi = bi;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float oc = __shfl_xor_sync(0xffffffffu, wc, off);
            const int oi = __shfl_xor_sync(0xffffffffu, wi, off);
            if (route_better(oc, oi, wc, wi)) {
                wc = oc;
                wi = oi;
            }
        }
        // the owner marks it and hands its affinity to lane j
        float ws = 0.f;
        if (wi == bi && bslot >= 0) {
            taken |= 1u << bslot;
            ws = route_sigmoid(u[wi]);
        }
        ws = __shfl_sync(0xffffffffu, ws, wi & 31);
        if (lane == j) {
            id = wi;
            s_out = ws;
        }
    }
}

}  // namespace fg8
