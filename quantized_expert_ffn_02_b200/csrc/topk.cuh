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
    int e;       // lane r < k: the rank-r expert (-1 if adaptive top-p dropped it)
    float w;     // its gate weight (fp64 arithmetic, rounded once; 0 if dropped)
    int pos;     // its position among the k entries in ascending (expert, rank) order
};

// Gate weights of the chosen experts and their positions in ascending index order.  Lane r < k
// holds the rank-r expert e and its logit l (fp64 arithmetic, rounded once to fp32).
__device__ __forceinline__ TopkPick topk_finish(int my_e, double my_l, int k, int router, float scaling, int lane,
                                                double top_p = 0.0) {
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
    double w = mine ? (double)scaling * num / den : 0.0;
    if (top_p > 0.0 && top_p < 1.0) {
        // the k weights' total and running share, in rank order (every lane walks the same sums)
        double total = 0.0;
        for (int r2 = 0; r2 < k; ++r2) total += __shfl_sync(0xffffffffu, w, r2);
        // the running share in rank order; the kept total is that prefix sum where it stops
        double cum = 0.0, kept = 0.0;
        int m = k;
        for (int r2 = 0; r2 < k; ++r2) {
            cum += __shfl_sync(0xffffffffu, w, r2);
            if (cum / total >= top_p) {
                m = r2 + 1;
                break;
            }
        }
        kept = cum;
        if (lane < m) {
            w = w * (total / kept);
        } else if (mine) {
            w = 0.0;
            my_e = -1;
        }
    }
    int pos = 0;
    for (int r2 = 0; r2 < k; ++r2) {
        const int e2 = __shfl_sync(0xffffffffu, my_e, r2);
        if (mine && (e2 < my_e || (e2 == my_e && r2 < lane))) ++pos;
    }
    TopkPick p;
    p.e = mine ? my_e : -1;
    p.w = mine ? (float)w : 0.0f;
    p.pos = pos;
    return p;
}

// An fp64 key as an unsigned integer of the same order (-0 folded into +0; NaN is not passed),
// never 0, so that 0 can stand for "none"; and back.
__device__ __forceinline__ unsigned long long key_order(double v) {
    const long long b = __double_as_longlong(v + 0.0);
    return b < 0 ? ~(unsigned long long)b : (unsigned long long)b | (1ull << 63);
}
__device__ __forceinline__ double key_value(unsigned long long o) {
    return __longlong_as_double((long long)(o >> 63 ? o & ~(1ull << 63) : ~o));
}
// The warp-wide largest of the lanes' order-mapped values: two single-instruction reductions.
__device__ __forceinline__ unsigned long long warp_max_order(unsigned long long v) {
    const unsigned hi = (unsigned)(v >> 32), mh = __reduce_max_sync(0xffffffffu, hi);
    const unsigned lo = hi == mh ? (unsigned)v : 0u, ml = __reduce_max_sync(0xffffffffu, lo);
    return ((unsigned long long)mh << 32) | ml;
}

// Group-limited selection: marks (in `taken`) every expert outside the topk_group best groups.
// ok[m] is the order-mapped key of expert lane + 32 m.  n_group <= 32 and E % n_group == 0.
template <int MAXPER>
__device__ __forceinline__ void limit_groups(const unsigned long long (&ok)[MAXPER], int E, const RouterOpts& o,
                                             int lane, uint32_t& taken) {
    const int G = o.n_group, per = E / G;
    double my_score = -INFINITY;             // lane g: the score of group g
    for (int g = 0; g < G; ++g) {
        // this lane's two largest keys of the group (l1 >= l2), then the group's: the largest,
        // and the largest once the lowest-indexed holder of the largest is set aside
        unsigned long long l1 = 0ull, l2 = 0ull;
        int i1 = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m) {
            const int e = lane + kWarp * m;
            if (e < E && e / per == g) {
                if (ok[m] > l1) { l2 = l1; l1 = ok[m]; i1 = e; }
                else if (ok[m] > l2) l2 = ok[m];
            }
        }
        const unsigned long long m1 = warp_max_order(l1);
        const unsigned w1 = __reduce_min_sync(0xffffffffu, l1 == m1 ? (unsigned)i1 : 0xffffffffu);
        const unsigned long long m2 = warp_max_order((unsigned)i1 == w1 ? l2 : l1);
        if (lane == g) my_score = per >= 2 ? key_value(m1) + key_value(m2) : key_value(m1);
    }
    // the topk_group best groups (ties to the lower group)
    const unsigned long long so = lane < G ? key_order(my_score) : 0ull;
    uint32_t keep = 0;
    for (int r = 0; r < o.topk_group; ++r) {
        const bool open = lane < G && !(keep >> lane & 1u);
        const unsigned long long mx = warp_max_order(open ? so : 0ull);
        keep |= 1u << __reduce_min_sync(0xffffffffu, open && so == mx ? (unsigned)lane : 0xffffffffu);
    }
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
        const int e = lane + kWarp * m;
        if (e < E && !(keep >> (e / per) & 1u)) taken |= 1u << m;
    }
}

// The selection key of one expert: the logit (softmax router) or sigmoid(logit) + bias; NaN
// never wins.
__device__ __forceinline__ double topk_key(double l, float bias, int router) {
    const double kv = router == MOE_ROUTER_SIGMOID_BIAS ? 1.0 / (1.0 + exp(-l)) + (double)bias : l;
    return isnan(kv) ? -INFINITY : kv;
}

// key[m] and lg[m] are the selection key (topk_key) and the logit of expert lane + 32 m; entries
// with an index >= E are ignored.  Every lane of the warp calls it; lanes >= k get e = -1.
template <int MAXPER>
__device__ __forceinline__ TopkPick warp_topk_keys(double (&key)[MAXPER], const double (&lg)[MAXPER], int E, int k,
                                                   int router, float scaling, int lane, const RouterOpts& opts) {
    uint32_t taken = 0;
#pragma unroll
    for (int m = 0; m < MAXPER; ++m)
        if (lane + kWarp * m >= E) {
            taken |= 1u << m;
            key[m] = -INFINITY;
        }
    // Keys as unsigned integers of the same order (the keys are never NaN), so that each round's
    // warp-wide arg-max is three single-instruction reductions: the largest high word, then the
    // largest low word among the lanes holding that high word, then the smallest index among the
    // lanes holding the whole largest key.  0 stands for "none left".
    unsigned long long ok[MAXPER];
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) ok[m] = key_order(key[m]);
    if (opts.n_group > 1) limit_groups<MAXPER>(ok, E, opts, lane, taken);
    int my_e = -1;
    double my_l = 0.0;
    for (int r = 0; r < k; ++r) {
        unsigned long long bo = 0ull;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m)              // a lane's experts come in ascending index
            if (!(taken >> m & 1u) && ok[m] > bo) { bo = ok[m]; bi = lane + kWarp * m; }
        const unsigned long long mx = warp_max_order(bo);
        bi = (int)__reduce_min_sync(0xffffffffu, bo == mx ? (unsigned)bi : 0xffffffffu);
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
    return topk_finish(my_e, my_l, k, router, scaling, lane, opts.top_p);
}

// The same from the logits: lg[m] is the logit of expert lane + 32 m and bv[m] its selection bias
// (0 without one).
template <int MAXPER>
__device__ __forceinline__ TopkPick warp_topk(const double (&lg)[MAXPER], const float (&bv)[MAXPER], int E, int k,
                                              int router, float scaling, int lane,
                                              const RouterOpts& opts = RouterOpts()) {
    double key[MAXPER];
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) key[m] = lane + kWarp * m < E ? topk_key(lg[m], bv[m], router) : -INFINITY;
    return warp_topk_keys<MAXPER>(key, lg, E, k, router, scaling, lane, opts);
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
