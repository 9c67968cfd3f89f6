// decode_fused.cu -- the whole layer for one token with int4 experts, in one cooperative launch.
//
// For one token the layer reads each weight byte once, so its time is the time to stream the
// router matrix and k + 1 experts from HBM.  Separate kernels for the router, gate/up and down
// each pay the ramp of a fresh grid and leave HBM idle while the previous grid drains; here one
// persistent CTA per SM runs the three steps back to back and keeps its copies in flight across
// the joins:
//
//   A  router + shared expert.  Every warp first queues its shared-expert gate/up row pairs (they
//      need no routing) into its ring of TMA stages, then computes its piece of the router logits
//      (fp64, one expert x 1024 columns per unit) and stores it.  The CTA arrives on a grid
//      barrier, and the warps reduce their shared rows while the other CTAs arrive.
//   B  selection.  Warp 0 of every CTA waits for the barrier, sums the pieces (the same order in
//      every CTA, so every CTA selects the same experts) and runs the top-k; the k experts and
//      gate weights go to shared memory.
//   C  routed gate/up: row pairs of the k experts, h = SiLU(gate) * up in fp16 (global, L2).
//      A warp that has finished its row pairs queues its first down rows (they do not depend on h),
//      then the CTA arrives on the second grid barrier, after which every h is complete.
//   D  down + combine: CTA b owns output rows [b d / G, (b + 1) d / G) of every slot (the k
//      routed experts in ascending index order, then the shared expert); its warps split the
//      (slot, row) list, and the CTA adds the slots with their gate weights and stores y.
//
// Dequantisation and the precision of each step are those of decode1.cu (bf16 136 + s for
// gate/up with the offset removed through the sum of x; exact fp16 s for down; fp32
// accumulation; h rounded to fp16).  The router logits accumulate in fp64.
//
// The grid barrier counts arrivals in a 64-bit word that only grows.  Every CTA arrives exactly
// once at each of the two barriers of a launch, also on its error paths, so a launch starts with
// the count at a multiple of 2G (G = CTAs): the first arrival of a CTA returns a value in
// [2Gn, 2Gn + G), from which the CTA takes the base 2Gn; barrier b is complete when the count
// reaches 2Gn + (b + 1) G.  Every wait is bounded by a clock limit; a warp that gives up latches
// MOE_ERR_TIMEOUT, waits (bounded) for the copies it issued, still arrives where the others
// expect it, and skips the rest of its work.
#include "decode_common.cuh"
#include "topk.cuh"

#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace qe {
namespace {

using namespace dec;

constexpr int kFzMaxWarps = 12;
constexpr int kFzStages = 3;
constexpr int kFzMaxSlots = 10;       // k routed experts + the shared one
constexpr int kFzMaxPer = 8;          // experts per lane in the selection: E <= 256
constexpr int kFzRowsMax = 64;        // output rows per CTA
constexpr int kFzDnRowsMax = 8;       // down rows per stage
constexpr size_t kSmemLimit = 227 * 1024;
constexpr int kStaticReserve = 4096;  // static shared memory of the kernel, rounded up

struct FusedArgs {
    const float* router_w;            // [E][d] fp32
    const float* bias;                // [E] selection bias (sigmoid router) or null
    const uint16_t* x;                // [d] bf16
    const uint8_t* gate_up;           // [E][2f][d/2]
    const float* gu_scale;            // [E][2f]
    const uint8_t* sh_gate_up;        // [2f][d/2]
    const float* sh_gu_scale;         // [2f]
    const uint8_t* down;              // [E][d][f/2]
    const float* dn_scale;            // [E][d]
    const uint8_t* sh_down;           // [d][f/2]
    const float* sh_dn_scale;         // [d]
    double* rpart;                    // [E][d/1024] pieces of the router logits
    uint16_t* h;                      // [k+1][f] fp16
    void* out;                        // [d] fp32 or bf16
    int32_t* idx;                     // tables written by CTA 0 (the layer's debug reads)
    float* wts;
    int32_t* asc;
    int32_t* ulist;
    int32_t* n_unique;
    double* xsum;
    unsigned long long* bar;          // grid-barrier arrivals (never reset between launches)
    unsigned long long* trace;        // [CTA][8] %globaltimer at the phase boundaries
    int* status;
    int d, f, E, k, S, router, out_bf16, dn_rows;
    float scaling;
};

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// Arrive: this CTA's earlier writes (ordered before by __syncthreads) become visible first.
// Returns the count before the arrival.  One thread calls it.
__device__ __forceinline__ unsigned long long arrive(unsigned long long* count) {
    __threadfence();
    return atomicAdd(count, 1ull);
}
// Bounded wait until the arrival count reaches `target`.  One thread calls it.
__device__ bool wait_arrivals(const unsigned long long* count, unsigned long long target) {
    if (ld_acquire(count) >= target) return true;
    const uint64_t t0 = now_ns();
    while (ld_acquire(count) < target) {
        if (now_ns() - t0 > kWaitLimitNs) return false;
        __nanosleep(64);
    }
    return true;
}
__device__ __forceinline__ float4 ld_stream16f(const float* p) {
    const uint4 v = ld_stream16(p);
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}
// Start an L2 prefetch of [p, p + bytes) (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// 32 fp32 router weights (8 float4) of one lane.
__device__ __forceinline__ void load_router32(const float* w, float4 (&rw)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) rw[i] = ld_stream16f(w + 4 * i);
}
// x (32 bf16 columns at 8m .. 8m + 7 per group, paired as in pair_cols) dotted with the lane's 32
// router weights, in fp64.
__device__ __forceinline__ double router_piece(const float4 (&rw)[8], const uint32_t* xp) {
    double a = 0.0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 lo = rw[2 * m], hi = rw[2 * m + 1];
        const float wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t p = xp[4 * m + i];            // (column 8m + i, column 8m + i + 4)
            a = fma((double)__uint_as_float(p << 16), (double)wl[i], a);
            a = fma((double)__uint_as_float(p & 0xffff0000u), (double)wh[i], a);
        }
    }
    return a;
}

// Dot products of one gate row and one up row (stage at shared address st) with x.
template <int NCH>
__device__ __forceinline__ float2 gu_dot(uint32_t st, uint32_t gu_row, int lane, const uint32_t (&xr)[NCH][16]) {
    float ag = 0.0f, au = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const uint32_t off = (uint32_t)(lane + kWarp * j) * 16;
        const uint4 Gv = lds16(st + off), Uv = lds16(st + gu_row + off);
        ag = dot_word_bf16(Gv.x, &xr[j][0], ag);
        au = dot_word_bf16(Uv.x, &xr[j][0], au);
        ag = dot_word_bf16(Gv.y, &xr[j][4], ag);
        au = dot_word_bf16(Uv.y, &xr[j][4], au);
        ag = dot_word_bf16(Gv.z, &xr[j][8], ag);
        au = dot_word_bf16(Uv.z, &xr[j][8], au);
        ag = dot_word_bf16(Gv.w, &xr[j][12], ag);
        au = dot_word_bf16(Uv.w, &xr[j][12], au);
    }
    return make_float2(ag, au);
}

// NCH = d / 1024 (x chunks per lane), NCF = f / 1024 (h chunks per lane).
template <int NCH, int NCF>
__global__ void __launch_bounds__(kFzMaxWarps * kWarp, 1) decode_fused_kernel(const FusedArgs a) {
    // [kFzStages][warps][stage]: stage s of every warp is one contiguous region
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kFzMaxWarps][kFzStages];
    __shared__ __align__(8) uint64_t s_xbar;              // x -> shared memory
    __shared__ __align__(8) uint64_t s_rbar;              // the router pieces -> shared memory
    __shared__ float ys[kFzMaxSlots][kFzRowsMax];
    __shared__ int s_e[kFzMaxSlots];                       // routed experts, ascending
    __shared__ float s_w[kFzMaxSlots];                     // their gate weights
    __shared__ int sel_e[kFzMaxSlots];                     // rank order
    __shared__ double sel_l[kFzMaxSlots];
    __shared__ unsigned long long s_base;                 // arrivals before this launch
    __shared__ int s_ok;

    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int nwc = blockDim.x / kWarp;
    const int gw = blockIdx.x * nwc + warp, nw = gridDim.x * nwc;
    const int G = gridDim.x;
    const int d = a.d, f = a.f, k = a.k, E = a.E;
    const uint32_t gu_row = (uint32_t)d / 2, dn_row = (uint32_t)f / 2;
    const uint32_t stage_bytes = 2 * gu_row + 32;
    const uint32_t smem0 = saddr(smem);
    auto st_s = [&](int s) { return smem0 + ((uint32_t)s * nwc + warp) * stage_bytes; };
    auto st_g = [&](int s) { return smem + ((size_t)s * nwc + warp) * stage_bytes; };
    const int n_sh = a.S ? f : 0;                          // shared row pairs
    const int n_tasks = n_sh + k * f;
    auto count_of = [&](int lo, int hi) {                  // my tasks among [lo, hi)
        const int first = lo + ((gw - lo) % nw + nw) % nw; // smallest t >= lo with t == gw (mod nw)
        return first < hi ? (hi - first + nw - 1) / nw : 0;
    };
    const int my_sh = count_of(0, n_sh);
    const int my_tasks = my_sh + count_of(n_sh, n_tasks);
    // task i of this warp is t = gw + i * nw (shared ones first because gw < nw)
    // this CTA's output rows and the warp's share of the (slot, row) items
    const int j0 = (int)((int64_t)blockIdx.x * d / G), rj = (int)((int64_t)(blockIdx.x + 1) * d / G) - j0;
    const int nslots = k + a.S;
    const int n_items = nslots * rj;
    const int it0 = (int)((int64_t)warp * n_items / nwc), it1 = (int)((int64_t)(warp + 1) * n_items / nwc);

    unsigned long long* trace = a.trace + (size_t)blockIdx.x * kTraceStamps;
    auto stamp = [&](int i) {
        if (tid == 0) trace[i] = now_ns();
    };
    stamp(0);
    if (lane == 0) {
        for (int s = 0; s < kFzStages; ++s) bar_init(saddr(&bars[warp][s]), 1);
        if (warp == 0) {
            bar_init(saddr(&s_xbar), 1);
            bar_init(saddr(&s_rbar), 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // x (2d bytes) into the stage-2 region, once per CTA
    const uint32_t xs_s = smem0 + 2u * nwc * stage_bytes;
    if (tid == 0) {
        bar_expect_tx(saddr(&s_xbar), 2u * d);
        bulk_g2s(xs_s, a.x, 2u * d, saddr(&s_xbar));
    }

    // ---- the ring: use q of this warp goes to stage q % kFzStages
    //      q < my_tasks: gate/up row pair (task q); q >= my_tasks: down stage (items from dit)
    int issued = 0;               // lane 0: next use to issue
    int dit = it0;                // lane 0: first item of the next down stage to issue
    auto sliver = [](const float* p) { return reinterpret_cast<const float*>((uintptr_t)p & ~(uintptr_t)15); };
    auto gu_src = [&](int i, const uint8_t*& rows, const float*& sc, int& r, int& slot) {
        const int t = gw + i * nw;
        if (t < n_sh) {
            rows = a.sh_gate_up + (size_t)t * gu_row;
            sc = a.sh_gu_scale + t;
            r = t;
            slot = k;
        } else {
            const int t2 = t - n_sh, u = t2 / f;
            r = t2 - u * f;
            const size_t row = (size_t)s_e[u] * 2 * f + r;
            rows = a.gate_up + row * gu_row;
            sc = a.gu_scale + row;
            slot = u;
        }
    };
    auto dn_stage = [&](int it, int& u, int& row, int& n) {  // stage starting at item `it`
        u = it / rj;
        row = it - u * rj;
        n = min(min(a.dn_rows, it1 - it), rj - row);
    };
    auto issue = [&](int q) {
        const uint32_t bar = saddr(&bars[warp][q % kFzStages]);
        const uint32_t dst = st_s(q % kFzStages);
        if (q < my_tasks) {
            const uint8_t* rows;
            const float* sc;
            int r, slot;
            gu_src(q, rows, sc, r, slot);
            bar_expect_tx(bar, stage_bytes);
            bulk_g2s(dst, rows, gu_row, bar);
            bulk_g2s(dst + gu_row, rows + (size_t)f * gu_row, gu_row, bar);
            bulk_g2s(dst + 2 * gu_row, sliver(sc), 16, bar);
            bulk_g2s(dst + 2 * gu_row + 16, sliver(sc + f), 16, bar);
        } else {
            int u, row, n;
            dn_stage(dit, u, row, n);
            const uint8_t* W = u < k ? a.down + (size_t)s_e[u] * d * dn_row : a.sh_down;
            bar_expect_tx(bar, (uint32_t)n * dn_row);
            bulk_g2s(dst, W + (size_t)(j0 + row) * dn_row, (uint32_t)n * dn_row, bar);
            dit += n;
        }
    };
    auto wait_use = [&](int q) {
        const bool ok = bar_wait(saddr(&bars[warp][q % kFzStages]), (uint32_t)(q / kFzStages) & 1u);
        return __all_sync(0xffffffffu, ok);
    };
    auto drain = [&](int from) {      // lane 0: let every copy still in flight land
        if (lane == 0)
            for (int q = from; q < issued; ++q)
                bar_wait(saddr(&bars[warp][q % kFzStages]), (uint32_t)(q / kFzStages) & 1u);
    };

    // ---- A: x (one bulk copy per CTA) and this warp's first router piece are fetched first, ahead
    //      of the stream of expert rows, so that the router's inputs are not queued behind it
    const int n_units = E * NCH;
    float4 rw[8];
    if (gw < n_units) {
        const int e = gw / NCH, p = gw - e * NCH;
        load_router32(a.router_w + (size_t)e * d + 1024 * p + 32 * lane, rw);
    }
    const float my_bias = a.bias && tid < E ? a.bias[tid] : 0.0f;
    bool ok = __all_sync(0xffffffffu, bar_wait(saddr(&s_xbar), 0u));
    // the shared expert's rows need no routing: queue them now (stages 0 and 1; stage 2 holds x)
    if (lane == 0)
        while (issued < my_sh && issued < kFzStages - 1) issue(issued++);
    // the shared expert's down rows of this CTA are read last: start pulling them into L2
    if (a.S && tid == kWarp && rj > 0)
        prefetch_l2(a.sh_down + (size_t)j0 * dn_row, (uint32_t)rj * dn_row);
    // x into registers (lane owns chunks lane + 32 j) and the sum of x
    uint32_t xr[NCH][16];
    float xsl = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + kWarp * j;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint4 v = lds16(xs_s + (uint32_t)(c * 32 + 8 * m) * 2u);
            pair_cols(v, &xr[j][4 * m]);
            const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                xsl += __uint_as_float(ws[q] << 16) + __uint_as_float(ws[q] & 0xffff0000u);
        }
    }
    const double xs = warp_sum_d((double)xsl);
    const float off136 = 136.0f * (float)xs;
    stamp(1);

    // router pieces: unit u = (expert u / NCH, columns [1024 p, 1024 p + 1024), p = u % NCH)
    for (int u = gw; u < n_units; u += nw) {
        const int e = u / NCH, p = u - e * NCH;
        if (u != gw) load_router32(a.router_w + (size_t)e * d + 1024 * p + 32 * lane, rw);
        double v = 0.0;
#pragma unroll
        for (int j = 0; j < NCH; ++j)
            if (j == p) v = router_piece(rw, xr[j]);
        v = warp_sum_d(v);
        if (lane == 0) __stcg(a.rpart + u, v);
    }
    __syncthreads();                                       // every warp has read x: stage 2 is free
    if (tid == 0) {                                        // barrier 0: every piece is stored
        const unsigned long long old = arrive(a.bar);
        s_base = old - old % (2ull * G);
    }
    stamp(2);

    // ---- one gate/up row pair: stage of use q -> h[slot][r]
    int limit = my_sh;            // lane 0: uses that may be issued so far
    auto gate_up_use = [&](int q, float2 acc) {
        const int s = q % kFzStages;
        const uint8_t* rows;
        const float* sc;
        int r, slot;
        gu_src(q, rows, sc, r, slot);
        const float* scs = reinterpret_cast<const float*>(st_g(s) + 2 * gu_row);
        const float sg = scs[(uintptr_t)sc / 4 & 3], su = scs[4 + ((uintptr_t)(sc + f) / 4 & 3)];
        __syncwarp();                                      // the stage is free again
        if (lane == 0)
            while (issued < limit && issued < q + 1 + kFzStages) issue(issued++);
        const float ag = warp_sum(acc.x), au = warp_sum(acc.y);
        if (lane == 0) {
            const float gv = sg * (ag - off136);
            const float uv = su * (au - off136);
            const float hv = gv / (1.0f + expf(-gv)) * uv;
            const __half hh = __float2half_rn(hv);
            if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(a.status, MOE_ERR_RANGE);
            a.h[(size_t)slot * f + r] = __half_as_ushort(hh);
        }
    };

    int q = 0;                    // next use to consume
    for (; ok && q < my_sh; ++q) {                         // the shared expert's row pairs
        if (lane == 0)
            while (issued < limit && issued < q + kFzStages) issue(issued++);
        if (!wait_use(q)) { ok = false; break; }
        gate_up_use(q, gu_dot<NCH>(st_s(q % kFzStages), gu_row, lane, xr));
    }

    // ---- B: selection by the whole CTA once every piece of the logits is stored.  The rings are
    //      idle: the router pieces, then the keys and logits, go to the start of shared memory.
    __syncthreads();
    stamp(3);
    const uint32_t rbytes = ((uint32_t)n_units * 8u + 15u) & ~15u;
    double* keys = reinterpret_cast<double*>(smem + rbytes);
    double* lgs = keys + E;
    if (tid == 0) {
        const bool bok = wait_arrivals(a.bar, s_base + (unsigned long long)G);
        if (bok) {
            bar_expect_tx(saddr(&s_rbar), rbytes);
            bulk_g2s(smem0, a.rpart, rbytes, saddr(&s_rbar));
        } else {
            latch_status(a.status, MOE_ERR_TIMEOUT);
        }
        s_ok = bok;
    }
    __syncthreads();
    stamp(4);
    bool sel = s_ok != 0;
    if (sel) {
        const bool landed = bar_wait(saddr(&s_rbar), 0u);
        if (landed && tid < E) {
            const double* rp = reinterpret_cast<const double*>(smem);
            double l = 0.0;
#pragma unroll
            for (int p = 0; p < NCH; ++p) l += rp[tid * NCH + p];
            lgs[tid] = l;
            keys[tid] = topk_key(l, my_bias, a.router);
        }
        sel = !__syncthreads_or(!landed);
        if (!sel && tid == 0) latch_status(a.status, MOE_ERR_TIMEOUT);
        stamp(5);
        // rank of expert tid in (key descending, index ascending); the first k are chosen
        if (sel && tid < E) {
            const double mk = keys[tid];
            int rank = 0;
            for (int j = 0; j < E; ++j) {
                const double kj = keys[j];
                rank += (kj > mk) | ((kj == mk) & (j < tid));
            }
            if (rank < k) {
                sel_e[rank] = tid;
                sel_l[rank] = lgs[tid];
            }
        }
        __syncthreads();
        if (sel && warp == 0) {
            const TopkPick pk = topk_finish(lane < k ? sel_e[lane] : -1, lane < k ? sel_l[lane] : 0.0, k, a.router,
                                            a.scaling, lane);
            if (lane < k) {
                s_e[pk.pos] = pk.e;
                s_w[pk.pos] = pk.w;
                if (blockIdx.x == 0) {
                    a.idx[lane] = pk.e;
                    a.wts[lane] = pk.w;
                    a.asc[pk.pos] = lane;
                    a.ulist[pk.pos] = pk.e;
                }
            }
            if (blockIdx.x == 0 && lane == 0) {
                *a.n_unique = k;
                *a.xsum = xs;
            }
        }
    }
    // the keys were written through the generic proxy; TMA writes into the same bytes come next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();              // s_e, s_w set; the rings may be used again
    stamp(6);
    const bool routed = sel;

    // ---- C: the routed row pairs; then the first down stages (independent of h)
    int n_dn = 0;                 // this warp's down stages
    for (int it = it0; it < it1;) {
        int u, row, n;
        dn_stage(it, u, row, n);
        it += n;
        ++n_dn;
    }
    if (ok && routed) {
        limit = my_tasks + n_dn;
        for (; q < my_tasks; ++q) {
            if (lane == 0)
                while (issued < limit && issued < q + kFzStages) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            gate_up_use(q, gu_dot<NCH>(st_s(q % kFzStages), gu_row, lane, xr));
        }
        if (ok && lane == 0)
            while (issued < limit && issued < q + kFzStages) issue(issued++);
    }

    // barrier 1: every h is stored
    __syncthreads();
    stamp(7);
    if (tid == 0) {
        arrive(a.bar);
        const bool bok = !routed || wait_arrivals(a.bar, s_base + 2ull * G);
        if (!bok) latch_status(a.status, MOE_ERR_TIMEOUT);
        s_ok = routed && bok;
    }
    stamp(8);
    __syncthreads();

    // ---- D: down rows of this CTA's output block, slot by slot
    if (ok && s_ok) {
        uint32_t hr[NCF][16];
        int cur_u = -1;
        for (int it = it0; it < it1; ++q) {
            int u, row, n;
            dn_stage(it, u, row, n);
            const float* scp = (u < k ? a.dn_scale + (size_t)s_e[u] * d : a.sh_dn_scale) + j0 + row;
            const float my_sc = lane < n ? __ldg(scp + lane) : 0.0f;
            if (u != cur_u) {                              // this slot's h (written by other CTAs)
#pragma unroll
                for (int j = 0; j < NCF; ++j) {
                    const int c = lane + kWarp * j;
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        pair_cols(ld_cg16(a.h + (size_t)u * f + (size_t)c * 32 + 8 * m), &hr[j][4 * m]);
                }
                cur_u = u;
            }
            if (lane == 0)
                while (issued < limit && issued < q + kFzStages) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            const uint32_t st = st_s(q % kFzStages);
            float acc[kFzDnRowsMax];
#pragma unroll
            for (int rr = 0; rr < kFzDnRowsMax; ++rr) {
                float v = 0.0f;
                if (rr < n) {
#pragma unroll
                    for (int j = 0; j < NCF; ++j) {
                        const uint4 wv = lds16(st + (uint32_t)rr * dn_row + (uint32_t)(lane + kWarp * j) * 16);
                        v = dot_word_f16(wv.x, &hr[j][0], v);
                        v = dot_word_f16(wv.y, &hr[j][4], v);
                        v = dot_word_f16(wv.z, &hr[j][8], v);
                        v = dot_word_f16(wv.w, &hr[j][12], v);
                    }
                }
                acc[rr] = v;
            }
            __syncwarp();
            if (lane == 0)
                while (issued < limit && issued < q + 1 + kFzStages) issue(issued++);
#pragma unroll
            for (int rr = 0; rr < kFzDnRowsMax; ++rr) {
                if (rr < n) {
                    const float v = warp_sum(acc[rr]);
                    const float srow = __shfl_sync(0xffffffffu, my_sc, rr);
                    if (lane == 0) ys[u][row + rr] = srow * v;
                }
            }
            it += n;
        }
    }
    if (!ok && lane == 0) latch_status(a.status, MOE_ERR_TIMEOUT);
    drain(q);                     // copies still in flight (only after a failed wait) land first
    __syncthreads();
    stamp(9);

    // ---- combine: routed slots in ascending expert order, then the shared expert
    if (s_ok) {
        for (int i = tid; i < rj; i += blockDim.x) {
            float o = 0.0f;
            for (int u = 0; u < k; ++u) o = fmaf(s_w[u], ys[u][i], o);
            if (a.S) o += ys[k][i];
            if (a.out_bf16)
                static_cast<__nv_bfloat16*>(a.out)[j0 + i] = __float2bfloat16_rn(o);
            else
                static_cast<float*>(a.out)[j0 + i] = o;
        }
    }
    stamp(10);
}

size_t fz_stage_bytes(const LayerDims& L) { return (size_t)L.d + 32; }
int fz_warps(const LayerDims& L) {
    const int w = (int)((kSmemLimit - kStaticReserve) / ((size_t)kFzStages * fz_stage_bytes(L)));
    return w > kFzMaxWarps ? kFzMaxWarps : w;
}
int fz_dn_rows(const LayerDims& L) {
    const int r = (int)(fz_stage_bytes(L) / (size_t)(L.f / 2));
    return r > kFzDnRowsMax ? kFzDnRowsMax : r;
}

template <int NCH, int NCF>
const void* fz_kernel() { return (const void*)decode_fused_kernel<NCH, NCF>; }

const void* fz_pick(const LayerDims& L) {
    const int nch = L.d / 1024, ncf = L.f / 1024;
#define QE_FZ(N)                                          \
    case N:                                               \
        return ncf == 1 ? fz_kernel<N, 1>() : fz_kernel<N, 2>();
    switch (nch) {
        QE_FZ(1) QE_FZ(2) QE_FZ(3) QE_FZ(4) QE_FZ(5) QE_FZ(6) QE_FZ(7) QE_FZ(8)
        default: return nullptr;
    }
#undef QE_FZ
}

}  // namespace

bool decode_fused_shape_ok(const LayerDims& L) {
    if (!(L.wkind == MOE_W_INT4_ROWSCALE && L.d % 1024 == 0 && L.d / 1024 >= 1 && L.d / 1024 <= 8 &&
          (L.f == 1024 || L.f == 2048) && (!L.S || L.f_shared == L.f) && L.k + L.S <= kFzMaxSlots &&
          L.E <= kWarp * kFzMaxPer && L.k <= L.E && fz_warps(L) >= 4 && fz_dn_rows(L) >= 1))
        return false;
    // the selection keeps the router pieces, keys and logits in the (idle) rings; E <= threads
    const size_t dyn = (size_t)fz_warps(L) * kFzStages * fz_stage_bytes(L);
    const size_t sel_bytes = ((size_t)L.E * (L.d / 1024) * 8 + 15) / 16 * 16 + 16 * (size_t)L.E;
    return sel_bytes <= dyn && L.E <= fz_warps(L) * kWarp;
}

cudaError_t prepare_decode_fused(const LayerDims& L, int num_sms, bool* usable) {
    *usable = false;
    if (!decode_fused_shape_ok(L) || (L.d + num_sms - 1) / num_sms > kFzRowsMax || num_sms > kTraceCtas)
        return cudaSuccess;
    int dev = 0, coop = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess || !coop) return e;
    const void* fn = fz_pick(L);
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    if (fa.sharedSizeBytes > (size_t)kStaticReserve) return cudaSuccess;
    const size_t dyn = (size_t)fz_warps(L) * kFzStages * fz_stage_bytes(L);
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(kSmemLimit - fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
    int blocks = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, fz_warps(L) * kWarp, dyn);
    if (e != cudaSuccess) return e;
    *usable = blocks >= 1;
    return cudaSuccess;
}

size_t decode_fused_rpart_count(const LayerDims& L) { return (size_t)L.E * (L.d / 1024 > 0 ? L.d / 1024 : 1); }

cudaError_t launch_decode_fused(const LayerDims& L, const moe_weights& W, const uint16_t* x, const Workspace& ws,
                                void* out, int num_sms, const Launch& ctx) {
    FusedArgs a;
    a.router_w = W.router_w;
    a.bias = L.router == MOE_ROUTER_SIGMOID_BIAS ? W.router_bias : nullptr;
    a.x = x;
    a.gate_up = (const uint8_t*)W.gate_up;
    a.gu_scale = W.gate_up_scale;
    a.sh_gate_up = (const uint8_t*)W.shared_gate_up;
    a.sh_gu_scale = W.shared_gate_up_scale;
    a.down = (const uint8_t*)W.down;
    a.dn_scale = W.down_scale;
    a.sh_down = (const uint8_t*)W.shared_down;
    a.sh_dn_scale = W.shared_down_scale;
    a.rpart = ws.rpart;
    a.h = ws.h;
    a.out = out;
    a.idx = ws.idx;
    a.wts = ws.wts;
    a.asc = ws.asc;
    a.ulist = ws.ulist;
    a.n_unique = ws.n_unique;
    a.xsum = ws.xsum;
    a.bar = ws.gbar;
    a.trace = ws.trace;
    a.status = ws.status;
    a.d = L.d;
    a.f = L.f;
    a.E = L.E;
    a.k = L.k;
    a.S = L.S;
    a.router = L.router;
    a.out_bf16 = L.out_bf16;
    a.dn_rows = fz_dn_rows(L);
    a.scaling = L.scaling;
    const int warps = fz_warps(L);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);
    cfg.blockDim = dim3((unsigned)(warps * kWarp));
    cfg.dynamicSmemBytes = (size_t)warps * kFzStages * fz_stage_bytes(L);
    cfg.stream = ctx.s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&a};
    prof_mark(ctx.prof, MOE_KERNEL_FUSED, true, ctx.s);
    cudaError_t e = cudaLaunchKernelExC(&cfg, fz_pick(L), args);
    prof_mark(ctx.prof, MOE_KERNEL_FUSED, false, ctx.s);
    if (e != cudaSuccess) return e;
    ++*ctx.launches;
    return cudaSuccess;
}

}  // namespace qe
