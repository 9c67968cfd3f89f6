// topk.cuh -- top-k expert selection and gate weights for one token, by one warp.
//
// Granite's router (softmax over the logits, then the k largest, renormalised over the chosen k)
// and the DeepSeek-V3 router (sigmoid scores; the k largest of score + bias, where the bias only
// selects; gate weights = chosen scores renormalised, times routed_scaling_factor) in one routine.
// Softmax is monotone, so the selection can run on the logits themselves.  Ties go to the lower
// expert index; a NaN key never wins, so every pick is a valid index.
#pragma once

#include <math.h>

#include "internal.cuh"

namespace qe {

__device__ __forceinline__ bool topk_beats(double ka, int ia, double kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

struct TopkPick {
    int e;       // lane r < k: the rank-r expert
    float w;     // its gate weight (fp64 arithmetic, rounded once)
    int pos;     // its position among the k experts in ascending index order
};

// Gate weights of the chosen experts and their positions in ascending index order.  Lane r < k
// holds the rank-r expert e and its logit l (fp64 arithmetic, rounded once to fp32).
__device__ __forceinline__ TopkPick topk_finish(int my_e, double my_l, int k, int router, float scaling, int lane) {
    const bool mine = lane < k;
    double num, den;
    if (router == MOE_ROUTER_SIGMOID_BIAS) {
        num = mine ? 1.0 / (1.0 + exp(-my_l)) : 0.0;
        den = warp_sum_d(num);
    } else {
        double m = mine ? my_l : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
        num = mine ? exp(my_l - m) : 0.0;
        den = warp_sum_d(num);
    }
    int pos = 0;
    for (int r2 = 0; r2 < k; ++r2) {
        const int e2 = __shfl_sync(0xffffffffu, my_e, r2);
        if (mine && e2 < my_e) ++pos;
    }
    TopkPick p;
    p.e = mine ? my_e : -1;
    p.w = mine ? (float)((double)scaling * num / den) : 0.0f;
    p.pos = pos;
    return p;
}

// The selection key of one expert: the logit (softmax router) or sigmoid(logit) + bias; NaN
// never wins.
__device__ __forceinline__ double topk_key(double l, float bias, int router) {
    const double kv = router == MOE_ROUTER_SIGMOID_BIAS ? 1.0 / (1.0 + exp(-l)) + (double)bias : l;
    return isnan(kv) ? -INFINITY : kv;
}

// lg[m] is the logit of expert lane + 32 m and bv[m] its selection bias (0 without one); entries
// with an index >= E are ignored.  Every lane of the warp calls it; lanes >= k get e = -1.
template <int MAXPER>
__device__ __forceinline__ TopkPick warp_topk(const double (&lg)[MAXPER], const float (&bv)[MAXPER], int E, int k,
                                              int router, float scaling, int lane) {
    double key[MAXPER];
    uint32_t taken = 0;
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
        const int e = lane + kWarp * m;
        double kv = -INFINITY;
        if (e < E) {
            kv = topk_key(lg[m], bv[m], router);
        } else {
            taken |= 1u << m;
        }
        key[m] = kv;
    }
    int my_e = -1;
    double my_l = 0.0;
    for (int r = 0; r < k; ++r) {
        double bk = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m) {
            const int e = lane + kWarp * m;
            if (!(taken >> m & 1u) && topk_beats(key[m], e, bk, bi)) { bk = key[m]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (topk_beats(ok, oi, bk, bi)) { bk = ok; bi = oi; }
        }
        // the owner of the winner marks it and hands its logit to lane r
        const int owner = bi % kWarp, wm = bi / kWarp;
        double wl = 0.0;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m)
            if (m == wm) wl = lg[m];
        if (owner == lane) taken |= 1u << wm;
        wl = __shfl_sync(0xffffffffu, wl, owner);
        if (lane == r) { my_e = bi; my_l = wl; }
    }
    return topk_finish(my_e, my_l, k, router, scaling, lane);
}

// The biases of experts lane + 32 m (0 where there is none).
template <int MAXPER>
__device__ __forceinline__ void load_bias(const float* __restrict__ bias, int E, int lane, float (&bv)[MAXPER]) {
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
        const int e = lane + kWarp * m;
        bv[m] = bias && e < E ? bias[e] : 0.0f;
    }
}

}  // namespace qe
