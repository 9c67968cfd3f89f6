// router.cu -- K2: router logits (fp64 accumulation) and top-k selection.
//
// Softmax top-k (Glacial, "What works": the Granite MoE layer) and the DeepSeek-V3-style
// sigmoid router with a selection-only bias and routed_scaling_factor (colibri README and
// iliria page, "What's implemented": noaux_tc).  Logits are accumulated in fp64: every
// product bf16 * fp32 is exact in fp64, so the only rounding is in the sums and the top-k
// boundary is decided at fp64 resolution.  Equal keys go to the lower expert index.
#include <algorithm>

#include "internal.cuh"
#include "topk.cuh"

namespace qe {
namespace {

constexpr int kRouterWarps = 8;      // experts per block
constexpr int kRouterTokens = 8;     // tokens per block (x tile in shared memory)

// grid = (ceil(E / 8), ceil(T / 8)); one warp per expert row, 8 tokens per block.
// The block's x tile [8][d] bf16 sits in dynamic shared memory.  Blocks with
// blockIdx.x == 0 also write sum_i x[t][i] (fp64) for their tokens.
__global__ void __launch_bounds__(kRouterWarps * kWarp)
router_logits_kernel(const float* __restrict__ wr, const uint16_t* __restrict__ x, int T, int d, int E,
                     double* __restrict__ logits, double* __restrict__ xsum) {
    extern __shared__ __align__(16) uint16_t xs[];      // [kRouterTokens][d]
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    const int t0 = blockIdx.y * kRouterTokens;
    const int nt = min(kRouterTokens, T - t0);
    // stage x (16-byte copies; d % 64 == 0 so rows are 16-byte multiples)
    const int row16 = d / 8;
    for (int i = threadIdx.x; i < nt * row16; i += blockDim.x) {
        const int tt = i / row16, c = i % row16;
        reinterpret_cast<uint4*>(xs + (size_t)tt * d)[c] =
            ld_ro16(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * d) + c);
    }
    __syncthreads();
    if (blockIdx.x == 0 && warp < nt) {
        double acc = 0.0;
        for (int i = lane; i < d; i += kWarp) acc += (double)bf16_bits_to_f32(xs[(size_t)warp * d + i]);
        acc = warp_sum_d(acc);
        if (lane == 0) xsum[t0 + warp] = acc;
    }
    const int e = blockIdx.x * kRouterWarps + warp;
    if (e >= E) return;
    double acc[kRouterTokens];
#pragma unroll
    for (int tt = 0; tt < kRouterTokens; ++tt) acc[tt] = 0.0;
    const float4* wrow = reinterpret_cast<const float4*>(wr + (size_t)e * d);
    for (int c = lane; c < d / 4; c += kWarp) {
        const float4 wv = __ldg(wrow + c);
#pragma unroll
        for (int tt = 0; tt < kRouterTokens; ++tt) {
            if (tt < nt) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xs + (size_t)tt * d + 4 * c);
                acc[tt] = fma((double)__uint_as_float(xv.x << 16), (double)wv.x, acc[tt]);
                acc[tt] = fma((double)__uint_as_float(xv.x & 0xffff0000u), (double)wv.y, acc[tt]);
                acc[tt] = fma((double)__uint_as_float(xv.y << 16), (double)wv.z, acc[tt]);
                acc[tt] = fma((double)__uint_as_float(xv.y & 0xffff0000u), (double)wv.w, acc[tt]);
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < kRouterTokens; ++tt) {
        if (tt < nt) {
            const double v = warp_sum_d(acc[tt]);
            if (lane == 0) logits[(size_t)(t0 + tt) * E + e] = v;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Large batches: logits = X Wr^T as a tiled fp64 GEMM on the fp64 tensor cores (mma.sync
// m8n8k4.f64: the only tensor-core form with fp64 operands and accumulator).  A CTA computes
// 64 tokens x 64 experts; every x and w element is converted to fp64 once per tile (into shared
// memory, K-major, rows padded to 68 so that a fragment load meets no bank conflict); warp
// (wm, wn) of the 2 x 4 warp grid owns 32 tokens x 16 experts, i.e. 4 x 2 tiles of 8 x 8.  The
// next K chunk's global loads are in flight while the current chunk is multiplied.  CTAs of the
// first expert tile also write sum_i x[t][i].
//
// The K range may be split over gridDim.z CTAs (slice z covers [z d / Z, (z + 1) d / Z)): slice z
// writes its partial logits to logits + z T E and its partial sums of x to xsum + z T, and the
// top-k kernel adds the slices in slice order.  More CTAs keep every SM's FP64 pipe busy: with
// one slice a 2048-token batch has 128 CTAs for 148 SMs, each a long chain of dependent chunks.
// ---------------------------------------------------------------------------------------
constexpr int kRgT = 64, kRgE = 64, kRgK = 32, kRgThreads = 256;
constexpr int kRgSplitMax = 3;

__global__ void __launch_bounds__(kRgThreads)
router_gemm_kernel(const float* __restrict__ wr, const uint16_t* __restrict__ x, int T, int d, int E,
                   double* __restrict__ logits, double* __restrict__ xsum) {
    __shared__ double xs[kRgK][kRgT + 4];
    __shared__ double ws[kRgK][kRgE + 4];
    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int wm = warp / 4, wn = warp % 4;                // 32 tokens x 16 experts per warp
    const int g = lane / 4, tq = lane % 4;                 // fragment row / column group
    const int t0 = blockIdx.x * kRgT, e0 = blockIdx.y * kRgE;
    const int kz = d / (int)gridDim.z, kb = (int)blockIdx.z * kz;      // this CTA's K slice
    logits += (size_t)blockIdx.z * T * E;
    xsum += (size_t)blockIdx.z * T;
    // loader roles: 4 threads per token row (8 bf16 each) and per expert row (8 fp32 each)
    const int lr = tid / 4, lc = (tid % 4) * 8;
    const bool xrow_ok = t0 + lr < T;
    const bool sum_x = blockIdx.y == 0;
    const uint16_t* xrow = x + (size_t)(xrow_ok ? t0 + lr : 0) * d + kb + lc;
    const float* wrow = wr + (size_t)(e0 + lr) * d + kb + lc;
    uint4 xv = xrow_ok ? ld_ro16(xrow) : make_uint4(0, 0, 0, 0);
    float4 wa = __ldg(reinterpret_cast<const float4*>(wrow)), wb = __ldg(reinterpret_cast<const float4*>(wrow) + 1);
    double acc[4][2][2];                                   // [token tile][expert tile][c0, c1]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    double xpart = 0.0;
    for (int k0 = 0; k0 < kz; k0 += kRgK) {
        // convert the staged chunk into shared memory (K-major)
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double lo = (double)__uint_as_float(xw[q] << 16), hi = (double)__uint_as_float(xw[q] & 0xffff0000u);
            xs[lc + 2 * q][lr] = lo;
            xs[lc + 2 * q + 1][lr] = hi;
            if (sum_x) xpart += lo + hi;
        }
        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) ws[lc + q][lr] = (double)wv[q];
        __syncthreads();
        // next chunk's loads go out before this chunk is multiplied
        if (k0 + kRgK < kz) {
            xv = xrow_ok ? ld_ro16(xrow + k0 + kRgK) : make_uint4(0, 0, 0, 0);
            wa = __ldg(reinterpret_cast<const float4*>(wrow + k0 + kRgK));
            wb = __ldg(reinterpret_cast<const float4*>(wrow + k0 + kRgK) + 1);
        }
#pragma unroll
        for (int kk = 0; kk < kRgK; kk += 4) {
            // A fragment (8 x 4, row-major): lane (g, tq) holds A[g][tq]; B (4 x 8, column-major):
            // B[tq][g]; C (8 x 8): C[g][2 tq], C[g][2 tq + 1]
            double a[4], b[2];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[kk + tq][32 * wm + 8 * i + g];
#pragma unroll
            for (int j = 0; j < 2; ++j) b[j] = ws[kk + tq][16 * wn + 8 * j + g];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                                 : "+d"(acc[i][j][0]), "+d"(acc[i][j][1])
                                 : "d"(a[i]), "d"(b[j]));
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 32 * wm + 8 * i + g;
        if (t < T)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = e0 + 16 * wn + 8 * j + 2 * tq;
                logits[(size_t)t * E + e] = acc[i][j][0];
                logits[(size_t)t * E + e + 1] = acc[i][j][1];
            }
    }
    if (sum_x) {     // the 4 loader threads of a token are adjacent lanes
        xpart += __shfl_xor_sync(0xffffffffu, xpart, 1);
        xpart += __shfl_xor_sync(0xffffffffu, xpart, 2);
        if ((tid & 3) == 0 && xrow_ok) xsum[t0 + lr] = xpart;
    }
}

// One warp per token: top-k and gate weights.
// Writes idx[t][r] / w[t][r] in rank order and asc[t][p] = the rank whose expert is the
// p-th smallest of the token's k experts.  With nsplit > 1 the logits are the sum of nsplit K
// slices (slice z at logits + z T E, added in slice order), and xsum[t] is formed the same way
// from the slices at xpart.
template <int MAXPER>
__global__ void __launch_bounds__(256)
topk_kernel(const double* __restrict__ logits, int nsplit, const double* __restrict__ xpart, double* __restrict__ xsum,
            const float* __restrict__ bias, int T, int E, int k, int router, float scaling,
            int32_t* __restrict__ idx_out, float* __restrict__ w_out, int32_t* __restrict__ asc_out,
            const RouterOpts opts) {
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    const int t = blockIdx.x * (blockDim.x / kWarp) + warp;
    if (t >= T) return;
    double lg[MAXPER];
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
        const int e = lane + kWarp * m;
        double v = 0.0;
        if (e < E) {
            v = logits[(size_t)t * E + e];
            for (int z = 1; z < nsplit; ++z) v += logits[((size_t)z * T + t) * E + e];
        }
        lg[m] = v;
    }
    if (xpart && lane == 0) {
        double v = xpart[t];
        for (int z = 1; z < nsplit; ++z) v += xpart[(size_t)z * T + t];
        xsum[t] = v;
    }
    float bv[MAXPER];
    load_bias<MAXPER>(bias, E, lane, bv);
    const TopkPick p = warp_topk<MAXPER>(lg, bv, E, k, router, scaling, lane, opts);
    if (lane < k) {
        idx_out[(size_t)t * k + lane] = p.e;
        w_out[(size_t)t * k + lane] = p.w;
        if (asc_out) asc_out[(size_t)t * k + p.pos] = lane;
    }
}

// ---------------------------------------------------------------------------------------
// Small batches (T <= 32): one launch for logits, top-k, gate weights and bucketing.
//
// Block (g, z) of the (NG, KS) grid owns the 16 experts 16 g .. 16 g + 15 (one per warp) and
// the K slice z: columns [64 ns z, 64 ns (z + 1)).  It stages the slice of every token's x in
// shared memory once, keeps its warp's router-row slice in registers (lane l: the column pairs
// 64 i + 2 l), and writes fp64 partial logits [z][t][e] for 8 tokens per pass; a transposed
// shuffle reduction leaves each token's sum in four lanes.  The last block of a group to finish
// (a per-group counter) adds the KS partials of its experts in slice order and writes their
// logits and selection keys; the last group to finish (a second counter) selects and buckets
// every token, a warp per token.  Every sum has a fixed order, so the logits do not depend on
// which block finished first.
// ---------------------------------------------------------------------------------------
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / kWarp;      // experts per block
constexpr int kSmallMaxT = 32;
constexpr int kSmallMaxE = 1024;
constexpr int kSmallMaxSteps = 12;                      // 64-column steps per slice (the fp64 tiles fit)
constexpr int kSmallMaxSlices = 16;

struct SmallArgs {
    const float* wr;            // [E][d] fp32 router
    const float* bias;          // [E] selection bias or null
    const uint16_t* x;          // [T][d] bf16
    int T, d, E, k, router, ns; // ns: 64-column steps per slice
    float scaling;
    double* part;               // [KS][T][E] partial logits, then [KS][T] partial x sums
    unsigned int* gcnt;         // [NG] blocks of each group done (reset by the group's last block)
    unsigned int* counter;      // groups done (reset by the last group)
    double* logits;             // [T][E]
    double* keys;               // [T][E]
    double* xsum;               // [T]
    int32_t *idx, *asc, *cnt, *off, *perm, *slot_of, *ulist, *n_unique;
    float* wts;
    RouterOpts opts;
    unsigned long long* trace;  // [block][16] %globaltimer at the phase boundaries, or null
};

// Selection for one token whose logits and keys other blocks wrote (read through L2).
template <int MAXPER>
__device__ void warp_select(const double* __restrict__ lg, const double* __restrict__ ky, int E, int k, int router,
                            float scaling, int lane, int32_t* idx_out, float* w_out, int32_t* asc_out,
                            const RouterOpts& opts, int32_t* idx_sh) {
    double l[MAXPER], key[MAXPER];
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
        const int e = lane + kWarp * m;
        l[m] = e < E ? __ldcg(lg + e) : 0.0;
        key[m] = e < E ? __ldcg(ky + e) : -INFINITY;
    }
    const TopkPick p = warp_topk_keys<MAXPER>(key, l, E, k, router, scaling, lane, opts);
    if (lane < k) {
        idx_out[lane] = p.e;
        idx_sh[lane] = p.e;
        w_out[lane] = p.w;
        asc_out[p.pos] = lane;
    }
}

// The sum over the warp of eight per-lane values v[0..7], reduced by halves: afterwards lane l
// holds the total of v[4 b4 + 2 b3 + b2] (b = the bits of l), the same in the four lanes that
// share those bits.  Fixed order, so every run gives the same value.
__device__ __forceinline__ double warp_sum8_scatter(const double (&v)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    double r4[4], r2[2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const double keep = b4 ? v[j + 4] : v[j], send = b4 ? v[j] : v[j + 4];
        r4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const double keep = b3 ? r4[j + 2] : r4[j], send = b3 ? r4[j] : r4[j + 2];
        r2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    double s = (b2 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? r2[0] : r2[1], 4);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    return s;
}

template <int MAXPER>
__global__ void __launch_bounds__(kSmallThreads, 1) route_small_kernel(const SmallArgs a) {
    extern __shared__ __align__(16) uint32_t xsm[];   // [T][32 ns] bf16 pairs of the slice, then [8][32 ns] fp64 pairs
    __shared__ int s_cnt[kSmallMaxE], s_off[kSmallMaxE], s_scan[kSmallThreads];
    __shared__ int s_idx[kSmallMaxT * kWarp];        // the chosen experts (k <= 32), for the bucketing
    __shared__ int am_last;
    const int g = blockIdx.x, z = blockIdx.y, NG = gridDim.x, KS = gridDim.y;
    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int T = a.T, d = a.d, E = a.E, ns = a.ns;
    const int c0 = 64 * ns * z;                    // the slice's first column
    const int e = g * kSmallWarps + warp;          // this warp's expert
    unsigned long long* const tr = a.trace ? a.trace + (size_t)(z * NG + g) * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (tid == 0 && tr) {
            unsigned long long v;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(v));
            tr[i] = v;
        }
    };
    stamp(0);
    // A kernel launched after this one with programmatic dependent launch may start now: it
    // waits (griddepcontrol.wait) before it reads anything written here.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // ---- shared memory: x's slice for every token (bf16), then fp64 tiles: the group's 16
    //      router-row slices [16][kc + 4] and one pass's 8 token slices [8][kc + 4] (rows padded
    //      by 4 doubles so that each half-warp's fragment loads meet 32 distinct banks), then the
    //      warps' partial products [16][64]
    const int kc = 64 * ns, pitch = kc + 4;        // columns of the slice, row pitch (doubles)
    double* const wd = reinterpret_cast<double*>(xsm + (size_t)T * 32 * ns);
    double* const xd = wd + (size_t)kSmallWarps * pitch;
    double* const red = xd + (size_t)8 * pitch;
    for (int i = tid; i < kSmallWarps * (kc / 4); i += kSmallThreads) {     // the router slices, in fp64
        const int r = i / (kc / 4), c = i - r * (kc / 4);
        const int ee = g * kSmallWarps + r;
        const float4 v = ee < E ? __ldg(reinterpret_cast<const float4*>(a.wr + (size_t)ee * d + c0) + c)
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        double* const dst = wd + (size_t)r * pitch + 4 * c;
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
    }
    const int row16 = 8 * ns;                      // 16-byte groups of a token's slice
    for (int i = tid; i < T * row16; i += kSmallThreads) {
        const int t = i / row16, c = i - t * row16;
        reinterpret_cast<uint4*>(xsm)[i] = ld_ro16(reinterpret_cast<const uint4*>(a.x + (size_t)t * d + c0) + c);
    }
    __syncthreads();
    stamp(1);
    double* const xpart = a.part + (size_t)KS * T * E;     // [KS][T] partial sums of x
    if (g == 0) {                                  // the slice's x sums, one warp per token
        for (int t = warp; t < T; t += kSmallWarps) {
            double s = 0.0;
            for (int i = 0; i < ns; ++i) {
                const uint32_t v = xsm[(size_t)t * 32 * ns + 32 * i + lane];
                s += (double)__uint_as_float(v << 16) + (double)__uint_as_float(v & 0xffff0000u);
            }
            s = warp_sum_d(s);
            if (lane == 0) xpart[(size_t)z * T + t] = s;
        }
    }
    // ---- partial logits on the fp64 tensor cores (mma.sync m8n8k4), 8 tokens per pass: the
    //      block's 16 experts are two 8-expert tiles, and each tile's K slice is dealt to 8 warps
    //      (kc / 8 columns each); the 8 partial tiles are then added in warp order.
    const int tile = warp >> 3, kp = warp & 7, fg = lane >> 2, fq = lane & 3;
    const int kw = kc / 8;                         // columns per warp
    for (int t0 = 0; t0 < T; t0 += 8) {
        const int nt = min(8, T - t0);
        __syncthreads();                                   // the previous pass is done with xd, red
        for (int i = tid; i < 8 * (kc / 2); i += kSmallThreads) {      // x pairs of the pass, fp64
            const int j = i / (kc / 2), pr = i - j * (kc / 2);
            uint32_t v = 0u;                                // tokens past T: zeros (unused)
            if (j < nt) v = xsm[(size_t)(t0 + j) * 32 * ns + pr];
            double* const dst = xd + (size_t)j * pitch + 2 * pr;
            dst[0] = (double)__uint_as_float(v << 16);
            dst[1] = (double)__uint_as_float(v & 0xffff0000u);
        }
        __syncthreads();
        // A (8 x 4): lane (fg, fq) holds x[token fg][k + fq]; B (4 x 8): w[expert fg][k + fq];
        // C: tokens fg, experts 2 fq and 2 fq + 1 of the tile
        double c0v = 0.0, c1v = 0.0;
        const double* const xa = xd + (size_t)fg * pitch + kp * kw + fq;
        const double* const wb = wd + (size_t)(8 * tile + fg) * pitch + kp * kw + fq;
#pragma unroll 4
        for (int kk = 0; kk < kw; kk += 4)
            asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                         : "+d"(c0v), "+d"(c1v)
                         : "d"(xa[kk]), "d"(wb[kk]));
        red[(size_t)warp * 64 + 2 * lane] = c0v;
        red[(size_t)warp * 64 + 2 * lane + 1] = c1v;
        __syncthreads();
        if (tid < 128) {                                   // (tile, token, expert of the tile)
            const int tl = tid >> 6, o = tid & 63;         // o: the C element (lane o / 2, o % 2)
            double sum = 0.0;
#pragma unroll
            for (int p = 0; p < 8; ++p) sum += red[(size_t)(8 * tl + p) * 64 + o];
            const int tok = o >> 3, ex = 8 * tl + 2 * ((o >> 1) & 3) + (o & 1);
            const int t = t0 + tok, ee = g * kSmallWarps + ex;
            if (ee < E && t < T) a.part[((size_t)z * T + t) * E + ee] = sum;
        }
    }
    // ---- the last block of the group: logits and keys of its experts, slices added in order
    stamp(2);
    __threadfence();
    __syncthreads();
    if (tid == 0) am_last = atomicAdd(a.gcnt + g, 1u) == (unsigned)KS - 1u;
    __syncthreads();
    stamp(3);
    if (!am_last) return;
    __threadfence();
    for (int i = tid; i < T * kSmallWarps; i += kSmallThreads) {
        const int t = i / kSmallWarps, ee = g * kSmallWarps + (i - t * kSmallWarps);
        if (ee < E) {
            double pz[kSmallMaxSlices];                // every slice's load in flight, then the ordered sum
#pragma unroll
            for (int zz = 0; zz < kSmallMaxSlices; ++zz)
                pz[zz] = zz < KS ? __ldcg(a.part + ((size_t)zz * T + t) * E + ee) : 0.0;
            double s = 0.0;
#pragma unroll
            for (int zz = 0; zz < kSmallMaxSlices; ++zz)
                if (zz < KS) s += pz[zz];
            a.logits[(size_t)t * E + ee] = s;
            a.keys[(size_t)t * E + ee] = topk_key(s, a.bias ? a.bias[ee] : 0.0f, a.router);
        }
    }
    if (g == 0)
        for (int t = tid; t < T; t += kSmallThreads) {
            double pz[kSmallMaxSlices];
#pragma unroll
            for (int zz = 0; zz < kSmallMaxSlices; ++zz) pz[zz] = zz < KS ? __ldcg(xpart + (size_t)zz * T + t) : 0.0;
            double s = 0.0;
#pragma unroll
            for (int zz = 0; zz < kSmallMaxSlices; ++zz)
                if (zz < KS) s += pz[zz];
            a.xsum[t] = s;
        }
    if (tid == 0) a.gcnt[g] = 0u;
    stamp(4);
    // ---- the last group: select and bucket every token
    __threadfence();
    __syncthreads();
    if (tid == 0) am_last = atomicAdd(a.counter, 1u) == (unsigned)NG - 1u;
    __syncthreads();
    stamp(5);
    if (!am_last) return;
    __threadfence();
    const int k = a.k;
    for (int t = warp; t < T; t += kSmallWarps)
        warp_select<MAXPER>(a.logits + (size_t)t * E, a.keys + (size_t)t * E, E, k, a.router, a.scaling, lane,
                            a.idx + (size_t)t * k, a.wts + (size_t)t * k, a.asc + (size_t)t * k, a.opts,
                            s_idx + t * k);
    // Bucketing.  s_cnt[e] becomes the set of tokens that chose expert e (a bit per token:
    // T <= 32); its population is the count, and an entry's slot is its expert's offset plus
    // the number of earlier tokens in that set (stable, in token order).
    for (int i = tid; i < E; i += kSmallThreads) s_cnt[i] = 0;
    __syncthreads();
    stamp(6);
    for (int i = tid; i < T * k; i += kSmallThreads)
        if (s_idx[i] >= 0) atomicOr(reinterpret_cast<unsigned*>(&s_cnt[s_idx[i]]), 1u << (i / k));  // -1: dropped
    __syncthreads();
    stamp(7);
    // exclusive scan of (count, used) over the experts: each thread a run of experts, then a
    // warp scan and a scan of the warp totals
    const int per = (E + kSmallThreads - 1) / kSmallThreads;
    const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
    int sum = 0, used = 0;
    for (int i = e0; i < e1; ++i) {
        const int c = __popc((unsigned)s_cnt[i]);
        sum += c;
        used += c > 0;
    }
    const int mine = sum | (used << 16);     // T*k <= 1024 < 2^16 and E <= 1024 < 2^16
    int v = mine;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == kWarp - 1) s_scan[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kSmallWarps ? s_scan[lane] : 0;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kSmallWarps) s_scan[kSmallWarps + lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp ? s_scan[kSmallWarps + warp - 1] : 0);
    const int base = incl - mine;
    int run = base & 0xffff, urun = base >> 16;
    for (int i = e0; i < e1; ++i) {
        const int c = __popc((unsigned)s_cnt[i]);
        s_off[i] = run;
        a.cnt[i] = c;
        a.off[i] = run;
        if (c > 0) a.ulist[urun++] = i;
        run += c;
    }
    if (tid == kSmallThreads - 1) {
        a.off[E] = incl & 0xffff;
        *a.n_unique = incl >> 16;
    }
    __syncthreads();
    stamp(8);
    for (int i = tid; i < T * k; i += kSmallThreads) {
        const int ex = s_idx[i], t = i / k;
        int p = -1;                                        // -1: dropped by adaptive top-p
        if (ex >= 0) {
            p = s_off[ex] + __popc((unsigned)s_cnt[ex] & ((1u << t) - 1u));
            a.perm[p] = i;
        }
        a.slot_of[i] = p;
    }
    if (tid == 0) *a.counter = 0u;
    stamp(9);
}

// 64-column steps per K slice for a layer of width d and E experts: as many slices (at most 16)
// as give about one block per SM, each at most 16 steps; 0 if d does not allow it.
int small_steps(int d, int E, int num_sms) {
    const int steps = d / 64, ng = (E + kSmallWarps - 1) / kSmallWarps;
    if (d % 64 || steps < 1) return 0;
    const int want = std::max(1, std::min(kSmallMaxSlices, (num_sms + ng - 1) / ng));
    for (int ks = want; ks >= 1; --ks)
        if (steps % ks == 0 && steps / ks <= kSmallMaxSteps) return steps / ks;
    for (int ks = want + 1; ks <= kSmallMaxSlices; ++ks)
        if (steps % ks == 0 && steps / ks <= kSmallMaxSteps) return steps / ks;
    return 0;
}

}  // namespace

bool route_small_ok(const LayerDims& L, int num_sms) {
    return L.E <= kSmallMaxE && small_steps(L.d, L.E, num_sms) > 0;
}

size_t route_small_part_doubles(int E, int max_tokens) {
    const size_t t = (size_t)std::min(max_tokens, kSmallMaxT);
    return (size_t)kSmallMaxSlices * t * ((size_t)E + 1);
}

size_t route_small_groups(int E) { return (size_t)(E + kSmallWarps - 1) / kSmallWarps; }

cudaError_t launch_route_small(const LayerDims& L, const float* router_w, const float* router_bias, const uint16_t* x,
                               int T, const Workspace& ws, int num_sms, const Launch& ctx) {
    if (T == 0) return cudaSuccess;
    if (T > kSmallMaxT) return cudaErrorInvalidValue;
    const int ns = small_steps(L.d, L.E, num_sms);
    if (!ns || L.E > kSmallMaxE) return cudaErrorInvalidValue;
    SmallArgs a;
    a.wr = router_w;
    a.bias = L.router == MOE_ROUTER_SIGMOID_BIAS ? router_bias : nullptr;
    a.x = x;
    a.T = T;
    a.d = L.d;
    a.E = L.E;
    a.k = L.k;
    a.router = L.router;
    a.ns = ns;
    a.scaling = L.scaling;
    a.part = ws.rsmall;
    a.gcnt = ws.rsmall_cnt;
    a.counter = reinterpret_cast<unsigned int*>(ws.counter);
    a.logits = ws.logits;
    a.keys = ws.keys;
    a.xsum = ws.xsum;
    a.idx = ws.idx;
    a.asc = ws.asc;
    a.cnt = ws.cnt;
    a.off = ws.off;
    a.perm = ws.perm;
    a.slot_of = ws.slot_of;
    a.ulist = ws.ulist;
    a.n_unique = ws.n_unique;
    a.wts = ws.wts;
    a.opts = L.ropts;
    a.trace = L.phase_trace ? ws.trace : nullptr;
    const dim3 grid((unsigned)route_small_groups(L.E), (unsigned)(L.d / 64 / ns));
    // bf16 slices of every token, the fp64 router slices and one pass's fp64 x, the partial tiles
    const size_t smem = (size_t)T * 128 * ns + (size_t)(kSmallWarps + 8) * (64 * ns + 4) * 8 + 16 * 64 * 8;
#define QE_ROUTE_SMALL(MAXPER)                                                          \
    QE_LAUNCH(ctx, MOE_KERNEL_ROUTER_LOGITS,                                            \
              (route_small_kernel<MAXPER><<<grid, kSmallThreads, smem, ctx.s>>>(a)))
    if (L.E <= 32) QE_ROUTE_SMALL(1);
    else if (L.E <= 256) QE_ROUTE_SMALL(8);
    else QE_ROUTE_SMALL(32);
#undef QE_ROUTE_SMALL
    return cudaSuccess;
}

// The opt-in is set to the whole 227 KB once per device, so that layers of different widths
// can coexist; each launch still asks only for its own tile.
cudaError_t prepare_router(const LayerDims& L) {
    const size_t smem = (size_t)kRouterTokens * L.d * sizeof(uint16_t);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    // the small-batch router's x slices: at most 32 tokens x 16 steps x 128 bytes
    const int small = kSmallMaxT * kSmallMaxSteps * 128 + (kSmallWarps + 8) * (64 * kSmallMaxSteps + 4) * 8 + 16 * 64 * 8;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(route_small_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, small);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(route_small_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, small);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(route_small_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, small);
    return e;
}

size_t router_split_doubles(int E, int max_tokens) {
    if (max_tokens < kRgT || E % kRgE) return 0;
    return (size_t)kRgSplitMax * ((size_t)max_tokens * E + (size_t)max_tokens);
}

cudaError_t launch_router(const LayerDims& L, const float* router_w, const float* router_bias,
                          const uint16_t* x, int T, double* logits, double* xsum, int32_t* idx, float* wts,
                          int32_t* asc, const Launch& ctx, double* part, size_t part_doubles) {
    if (T == 0) return cudaSuccess;
    const cudaStream_t s = ctx.s;
    int nsplit = 1;
    const double* lg = logits;
    const double* xpart = nullptr;
    if (T >= kRgT && L.E % kRgE == 0 && L.d % kRgK == 0) {
        for (int z = kRgSplitMax; z > 1 && part; --z)
            if (L.d % (kRgK * z) == 0 && part_doubles >= (size_t)z * ((size_t)T * L.E + T)) {
                nsplit = z;
                break;
            }
        double* lg_dst = nsplit > 1 ? part : logits;
        double* xs_dst = nsplit > 1 ? part + (size_t)nsplit * T * L.E : xsum;
        lg = lg_dst;
        if (nsplit > 1) xpart = xs_dst;
        dim3 grid((unsigned)((T + kRgT - 1) / kRgT), (unsigned)(L.E / kRgE), (unsigned)nsplit);
        QE_LAUNCH(ctx, MOE_KERNEL_ROUTER_LOGITS,
                  (router_gemm_kernel<<<grid, kRgThreads, 0, s>>>(router_w, x, T, L.d, L.E, lg_dst, xs_dst)));
    } else {
        const size_t smem = (size_t)kRouterTokens * L.d * sizeof(uint16_t);
        dim3 grid((L.E + kRouterWarps - 1) / kRouterWarps, (T + kRouterTokens - 1) / kRouterTokens);
        QE_LAUNCH(ctx, MOE_KERNEL_ROUTER_LOGITS,
                  (router_logits_kernel<<<grid, kRouterWarps * kWarp, smem, s>>>(router_w, x, T, L.d, L.E, logits,
                                                                                  xsum)));
    }
    const int tpb = 8;
    const unsigned g = (unsigned)((T + tpb - 1) / tpb);
    const float* bias = L.router == MOE_ROUTER_SIGMOID_BIAS ? router_bias : nullptr;
    if (L.E <= 32)
        QE_LAUNCH(ctx, MOE_KERNEL_TOPK, (topk_kernel<1><<<g, tpb * kWarp, 0, s>>>(lg, nsplit, xpart, xsum, bias, T, L.E, L.k, L.router,
                                                                                    L.scaling, idx, wts, asc, L.ropts)));
    else if (L.E <= 256)
        QE_LAUNCH(ctx, MOE_KERNEL_TOPK, (topk_kernel<8><<<g, tpb * kWarp, 0, s>>>(lg, nsplit, xpart, xsum, bias, T, L.E, L.k, L.router,
                                                                                    L.scaling, idx, wts, asc, L.ropts)));
    else
        QE_LAUNCH(ctx, MOE_KERNEL_TOPK, (topk_kernel<32><<<g, tpb * kWarp, 0, s>>>(lg, nsplit, xpart, xsum, bias, T, L.E, L.k, L.router,
                                                                                     L.scaling, idx, wts, asc, L.ropts)));
    return cudaSuccess;
}

}  // namespace qe

// ---------------------------------------------------------------------------------------
// Routing for callers that cannot allocate device memory.
//
// Some callers of this library may not allocate on the device at all: code that runs while a
// CUDA graph is being captured (where an allocation call breaks the capture), engines that
// hand out every byte of device memory from their own preallocated arena, or real-time loops
// that forbid an allocation (and its implicit synchronisation) after start-up.  They can still
// route tokens with moe_route_noalloc: its only scratch (the fp64 logits and the per-token sum
// of x) lives in a fixed array inside this library's device image, which every GPU that loads
// the library holds until the process exits.
// ---------------------------------------------------------------------------------------
#include <mutex>

namespace qe {
namespace {

constexpr size_t kRouteScratchBytes = (size_t)1 << 20;       // 1 MiB per device
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the device object:
// kernels must be given the address that cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

std::mutex g_route_scratch_mu;
void* g_route_scratch_dev[kMaxDevices] = {};

// Set-up, once per device, with that device current: look up the array's device address and
// opt the router kernel into its shared memory.  Neither call allocates.
moe_status route_scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_route_scratch_mu);
    if (!g_route_scratch_dev[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        e = cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        g_route_scratch_dev[dev] = p;
    }
    *out = g_route_scratch_dev[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace qe

extern "C" moe_status moe_route_noalloc(const moe_config* cfg, const float* router_w, const float* router_bias,
                                        const uint16_t* x, int32_t T, int32_t* idx, float* w, moe_stream stream) {
    if (!cfg || T < 0) return MOE_ERR_INVALID_ARG;
    if (cfg->d <= 0 || cfg->d % 64 || cfg->d > 14336) return MOE_ERR_INVALID_ARG;
    if (cfg->n_experts < 1 || cfg->n_experts > 1024) return MOE_ERR_INVALID_ARG;
    if (cfg->top_k < 1 || cfg->top_k > cfg->n_experts || cfg->top_k > 32) return MOE_ERR_INVALID_ARG;
    if (cfg->router != MOE_ROUTER_SOFTMAX_TOPK && cfg->router != MOE_ROUTER_SIGMOID_BIAS) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!router_w || !x || !idx || !w) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)router_w & 15) || ((uintptr_t)x & 15) || ((uintptr_t)idx & 3) || ((uintptr_t)w & 3))
        return MOE_ERR_INVALID_ARG;
    // logits [T][E] fp64, then the sums of x [T] fp64, each part 256-byte aligned
    const size_t logits_bytes = ((size_t)T * cfg->n_experts * sizeof(double) + 255) & ~(size_t)255;
    const size_t need = logits_bytes + (size_t)T * sizeof(double);
    if (need > qe::kRouteScratchBytes) return MOE_ERR_UNSUPPORTED;
    cudaGetLastError();   // an error left pending by an earlier, unrelated call is not this call's
    void* scratch = nullptr;
    moe_status st = qe::route_scratch_for_current_device(&scratch);
    if (st != MOE_OK) return st;
    // Every byte the kernels read from the scratch is written earlier in the same call, so
    // nothing has to be cleared between calls.
    double* logits = static_cast<double*>(scratch);
    double* xsum = reinterpret_cast<double*>(static_cast<unsigned char*>(scratch) + logits_bytes);
    const qe::LayerDims L{cfg->d, cfg->f, cfg->n_experts, cfg->top_k, 0, 0, cfg->router, cfg->wkind, 0,
                          cfg->routed_scaling_factor};
    int launches = 0;
    const qe::Launch ctx{(cudaStream_t)stream, &launches, nullptr};
    const float* bias = cfg->router == MOE_ROUTER_SIGMOID_BIAS ? router_bias : nullptr;
    cudaError_t e = qe::launch_router(L, router_w, bias, x, T, logits, xsum, idx, w, nullptr, ctx, nullptr, 0);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
