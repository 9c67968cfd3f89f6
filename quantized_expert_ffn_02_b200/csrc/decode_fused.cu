// decode_fused.cu -- the whole layer for one token with int4 experts, in one cooperative launch.
//
// For one token the layer reads each weight byte once, so its time is the time to stream the
// router matrix and k + 1 experts from HBM.  Separate kernels for the router, gate/up and down
// each pay the ramp of a fresh grid and leave HBM idle while the previous grid drains; here one
// persistent CTA per SM (16 warps) runs the steps back to back and keeps its copies in flight
// across the joins.  Shared memory holds x, rearranged once per CTA so that a lane's 32-column
// chunk loads without bank conflicts, and one ring of two TMA stages per warp (a gate row, the
// matching up row and two 16-byte slivers holding their scales).
//
//   A  router + shared expert.  One bulk copy brings x in; each warp's first router piece (one
//      expert x 1024 columns, coalesced loads) is in flight meanwhile.  The warps rearrange x,
//      sum it, queue their shared-expert row pairs (they need no routing), compute their router
//      pieces in fp64 and store them.  The CTA arrives on grid barrier 0, and the warps reduce
//      their shared rows while the other CTAs arrive.
//   B  selection, by the whole CTA: one bulk copy gathers every piece; thread e sums expert e's
//      pieces (the same order in every CTA, so every CTA selects the same experts) and forms an
//      order-preserving integer key; the k best of each warp's 32 experts become candidates, and
//      each candidate's rank among the candidates is its overall rank.  The k experts (ascending)
//      and their gate weights go to shared memory.
//   C  routed gate/up: row pairs of the k experts, strided over every warp of the grid;
//      h = SiLU(gate) * up in fp16 (global, L2), the SiLU of 32 row pairs at a time.  A warp that
//      has finished its row pairs queues its first down rows (they do not depend on h), then the
//      CTA arrives on grid barrier 1, after which every h is complete.
//   D  down + combine: CTA b owns output rows [b d / G, (b + 1) d / G) of every slot (the k
//      routed experts in ascending index order, then the shared expert); its warps split the
//      (slot, row) list, and the CTA adds the slots with their gate weights and stores y.
//
// Dequantisation: gate/up as bf16 136 + s (one LOP3 per two codes) with the offset removed
// through the sum of x; down as fp16 3/2 + s/16 (one shift and one LOP3 per two codes) with the
// offset removed through the sum of h.  Products are exact, sums fp32, h is rounded to fp16; the
// router logits accumulate in fp64.
//
// Phase timestamps (%globaltimer, thread 0 of each CTA) go to the workspace for the layer's
// debug read.
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

constexpr int kFzMaxWarps = 16;
constexpr int kFzStages = 2;
constexpr int kFzMaxSlots = 10;       // k routed experts + the shared one
constexpr int kFzMaxPer = 8;          // experts per lane in the selection: E <= 256
constexpr int kFzRowsMax = 64;        // output rows per CTA
constexpr int kFzDnRowsMax = 8;       // down rows per stage
constexpr size_t kSmemLimit = 227 * 1024;
constexpr int kStaticReserve = 5120;  // static shared memory of the kernel, rounded up

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

// One lane's share of a 1024-column router piece: float4 number lane + 32 i (i < 8), so that each
// load instruction of the warp reads 512 contiguous bytes.
__device__ __forceinline__ void load_router_piece(const float* w, int lane, float4 (&rw)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) rw[i] = ld_stream16f(w + 4 * (lane + kWarp * i));
}
// The lane's part of the piece's dot product with x (bf16, plain order in shared memory at xs),
// in fp64.
__device__ __forceinline__ double router_piece(const float4 (&rw)[8], uint32_t xs, int lane) {
    double a = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t x01, x23;
        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x01), "=r"(x23) : "r"(xs + (uint32_t)(lane + kWarp * i) * 8u));
        a = fma((double)__uint_as_float(x01 << 16), (double)rw[i].x, a);
        a = fma((double)__uint_as_float(x01 & 0xffff0000u), (double)rw[i].y, a);
        a = fma((double)__uint_as_float(x23 << 16), (double)rw[i].z, a);
        a = fma((double)__uint_as_float(x23 & 0xffff0000u), (double)rw[i].w, a);
    }
    return a;
}

// x of one lane's chunk c (32 columns) from the pre-paired copy in shared memory: four 16-byte
// rows, the pairs (column 8m + i, column 8m + i + 4) for m = 0..3, i = 0..3.
__device__ __forceinline__ void load_xq(uint32_t xp_s, int nchunks, int c, uint32_t (&xq)[16]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint4 v = lds16(xp_s + (uint32_t)(m * nchunks + c) * 16u);
        xq[4 * m] = v.x;
        xq[4 * m + 1] = v.y;
        xq[4 * m + 2] = v.z;
        xq[4 * m + 3] = v.w;
    }
}

// Dot products of one gate row and one up row (stage at shared address st) with x; x comes from
// the pre-paired shared copy, so the loop over the lane's chunks stays rolled (a small loop body
// keeps the instruction cache warm).
__device__ __forceinline__ float2 gu_dot(uint32_t st, uint32_t gu_row, int lane, uint32_t xp_s, int nchunks) {
    // two accumulators per row (even and odd words) halve the chains of dependent FMAs
    float ag0 = 0.0f, ag1 = 0.0f, au0 = 0.0f, au1 = 0.0f;
#pragma unroll 2
    for (int c = lane; c < nchunks; c += kWarp) {
        uint32_t xq[16];
        load_xq(xp_s, nchunks, c, xq);
        const uint4 Gv = lds16(st + (uint32_t)c * 16), Uv = lds16(st + gu_row + (uint32_t)c * 16);
        ag0 = dot_word_bf16(Gv.x, &xq[0], ag0);
        au0 = dot_word_bf16(Uv.x, &xq[0], au0);
        ag1 = dot_word_bf16(Gv.y, &xq[4], ag1);
        au1 = dot_word_bf16(Uv.y, &xq[4], au1);
        ag0 = dot_word_bf16(Gv.z, &xq[8], ag0);
        au0 = dot_word_bf16(Uv.z, &xq[8], au0);
        ag1 = dot_word_bf16(Gv.w, &xq[12], ag1);
        au1 = dot_word_bf16(Uv.w, &xq[12], au1);
    }
    return make_float2(ag0 + ag1, au0 + au1);
}

// NCF = f / 1024 (h chunks per lane in the down phase).
template <int NCF>
__global__ void __launch_bounds__(kFzMaxWarps * kWarp, 1) decode_fused_kernel(const FusedArgs a) {
    // [x pre-paired: 2d bytes][kFzStages][warps][stage]: stage s of every warp is one region
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kFzMaxWarps][kFzStages];
    __shared__ int4 s_desc[kFzMaxWarps][kFzStages];       // gate/up stage: slot, row, scale slots
    __shared__ __align__(8) uint64_t s_xbar;              // x -> shared memory
    __shared__ __align__(8) uint64_t s_rbar;              // the router pieces -> shared memory
    __shared__ float ys[kFzMaxSlots][kFzRowsMax];
    __shared__ int s_e[kFzMaxSlots];                       // routed experts, ascending
    __shared__ float s_w[kFzMaxSlots];                     // their gate weights
    __shared__ int sel_e[kFzMaxSlots];                     // rank order
    __shared__ int cand_e[kFzMaxPer * kFzMaxSlots];       // selection candidates, k per warp
    __shared__ uint2 cand_k[kFzMaxPer * kFzMaxSlots];     // and their keys
    __shared__ double sel_l[kFzMaxSlots];
    __shared__ unsigned long long s_base;                 // arrivals before this launch
    __shared__ double s_xpart[kFzMaxWarps];                // sum of x per warp slice
    __shared__ int s_ok;

    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int nwc = blockDim.x / kWarp;
    const int gw = blockIdx.x * nwc + warp, nw = gridDim.x * nwc;
    const int G = gridDim.x;
    const int d = a.d, f = a.f, k = a.k, E = a.E;
    const int nchunks = d / 32, nch = d / 1024;
    const uint32_t gu_row = (uint32_t)d / 2, dn_row_b = (uint32_t)f / 2;
    const uint32_t stage_bytes = 2 * gu_row + 32;
    const uint32_t xp_s = saddr(smem);                     // x, pre-paired
    uint8_t* const rings = smem + 2 * d;
    const uint32_t rings_s = xp_s + 2u * d;
    auto st_s = [&](int s) { return rings_s + ((uint32_t)s * nwc + warp) * stage_bytes; };
    auto st_g = [&](int s) { return rings + ((size_t)s * nwc + warp) * stage_bytes; };
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
    // x (2d bytes) into the last stage's region, once per CTA
    const uint32_t xraw_s = st_s(kFzStages - 1) - (uint32_t)warp * stage_bytes;
    if (tid == 0) {
        bar_expect_tx(saddr(&s_xbar), 2u * d);
        bulk_g2s(xraw_s, a.x, 2u * d, saddr(&s_xbar));
    }

    // ---- the ring: use q of this warp goes to stage q % kFzStages
    //      q < my_tasks: gate/up row pair (task q); q >= my_tasks: down stage (lane 0's cursor)
    int issued = 0;               // lane 0: next use to issue
    int n_dn = 0;                 // this warp's down stages
    auto sliver = [](const float* p) { return reinterpret_cast<const float*>((uintptr_t)p & ~(uintptr_t)15); };
    // lane 0's cursors: the routed (slot, row) of its next routed row pair, the next down item
    int gu_u = -1, gu_r = 0;
    int dn_u = it0 / max(rj, 1), dn_row = it0 - dn_u * rj, dn_it = it0;
    auto dn_count = [&](int it, int row) { return min(min(a.dn_rows, it1 - it), rj - row); };
    auto issue = [&](int q) {
        const uint32_t bar = saddr(&bars[warp][q % kFzStages]);
        const uint32_t dst = st_s(q % kFzStages);
        if (q < my_tasks) {
            const int t = gw + q * nw;
            const uint8_t* rows;
            const float* sc;
            int r, slot;
            if (t < n_sh) {
                rows = a.sh_gate_up + (size_t)t * gu_row;
                sc = a.sh_gu_scale + t;
                r = t;
                slot = k;
            } else {
                if (gu_u < 0) {
                    gu_u = (t - n_sh) / f;
                    gu_r = t - n_sh - gu_u * f;
                }
                r = gu_r;
                slot = gu_u;
                const size_t row = (size_t)s_e[gu_u] * 2 * f + gu_r;
                rows = a.gate_up + row * gu_row;
                sc = a.gu_scale + row;
                for (gu_r += nw; gu_r >= f; gu_r -= f) ++gu_u;
            }
            // the consumer finds its row and, in the two 16-byte slivers, its two scales
            s_desc[warp][q % kFzStages] = make_int4(slot, r, (int)(((uintptr_t)sc >> 2) & 3),
                                                    4 + (int)(((uintptr_t)(sc + f) >> 2) & 3));
            bar_expect_tx(bar, stage_bytes);
            bulk_g2s(dst, rows, gu_row, bar);
            bulk_g2s(dst + gu_row, rows + (size_t)f * gu_row, gu_row, bar);
            bulk_g2s(dst + 2 * gu_row, sliver(sc), 16, bar);
            bulk_g2s(dst + 2 * gu_row + 16, sliver(sc + f), 16, bar);
        } else {
            const int n = dn_count(dn_it, dn_row);
            const uint8_t* W = dn_u < k ? a.down + (size_t)s_e[dn_u] * d * dn_row_b : a.sh_down;
            bar_expect_tx(bar, (uint32_t)n * dn_row_b);
            bulk_g2s(dst, W + (size_t)(j0 + dn_row) * dn_row_b, (uint32_t)n * dn_row_b, bar);
            dn_it += n;
            dn_row += n;
            if (dn_row == rj) {
                dn_row = 0;
                ++dn_u;
            }
        }
    };
    auto wait_use = [&](int q) {
        const bool ok = bar_wait(saddr(&bars[warp][q % kFzStages]), (uint32_t)(q / kFzStages) & 1u);
        __syncwarp();                                      // lane 0's stage descriptor is visible
        return __all_sync(0xffffffffu, ok);
    };
    auto drain = [&](int from) {      // lane 0: let every copy still in flight land
        if (lane == 0)
            for (int q = from; q < issued; ++q)
                bar_wait(saddr(&bars[warp][q % kFzStages]), (uint32_t)(q / kFzStages) & 1u);
    };

    // ---- A: x (one bulk copy per CTA) and this warp's first router piece, both ahead of the
    //      stream of expert rows, so that the router's inputs are not queued behind it
    const int n_units = E * nch;
    // this warp's first router piece: its loads (coalesced, 512 bytes per instruction) are in
    // flight while x lands and is rearranged
    float4 rw[8];
    if (gw < n_units) {
        const int e = gw / nch, p = gw - e * nch;
        load_router_piece(a.router_w + (size_t)e * d + 1024 * p, lane, rw);
    }
    bool ok = __all_sync(0xffffffffu, bar_wait(saddr(&s_xbar), 0u));
    stamp(11);
    // x pre-paired into its own region (group g = columns 8g .. 8g + 7 goes to row g % 4 of chunk
    // g / 4), and the sum of x: thread i adds groups i, i + threads, ... (fp32), each warp's
    // total goes to shared memory (fp64).
    {
        float xsl = 0.0f;
        for (int g = tid; g < d / 8; g += blockDim.x) {
            const uint4 v = lds16(xraw_s + (uint32_t)g * 16u);
            uint32_t p[4];
            pair_cols(v, p);
            sts16(xp_s + (uint32_t)((g & 3) * nchunks + (g >> 2)) * 16u, make_uint4(p[0], p[1], p[2], p[3]));
            const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) xsl += __uint_as_float(ws[i] << 16) + __uint_as_float(ws[i] & 0xffff0000u);
        }
        const double wsum = warp_sum_d((double)xsl);
        if (lane == 0) s_xpart[warp] = wsum;
    }
    // this thread's selection bias
    const float my_bias = a.bias && tid < E ? a.bias[tid] : 0.0f;
    __syncthreads();                                       // x is pre-paired
    stamp(1);
    // the shared expert's rows need no routing: queue them now (all stages but the last, which
    // keeps x in plain order for the router pieces)
    if (lane == 0)
        while (issued < my_sh && issued < kFzStages - 1) issue(issued++);
    // the shared expert's down rows of this CTA are read last: start pulling them into L2
    if (a.S && tid == kWarp && rj > 0)
        prefetch_l2(a.sh_down + (size_t)j0 * dn_row_b, (uint32_t)rj * dn_row_b);
    double xs = 0.0;                                       // sum of x, the same order in every warp
    for (int w = 0; w < nwc; ++w) xs += s_xpart[w];
    const float off136 = 136.0f * (float)xs;

    // router pieces: unit u = (expert u / nch, columns [1024 p, 1024 p + 1024), p = u % nch)
    for (int u = gw; u < n_units; u += nw) {
        const int e = u / nch, p = u - e * nch;
        if (u != gw) load_router_piece(a.router_w + (size_t)e * d + 1024 * p, lane, rw);
        const double v = warp_sum_d(router_piece(rw, xraw_s + 2048u * p, lane));
        if (lane == 0) __stcg(a.rpart + u, v);
    }
    __syncthreads();                                       // the last stage is free
    if (tid == 0) {                                        // barrier 0: every piece is stored
        const unsigned long long old = arrive(a.bar);
        s_base = old - old % (2ull * G);
    }
    stamp(2);

    // ---- one gate/up row pair: stage of use q.  Lane n of the warp keeps the n-th pending result
    //      (g, u, index into h); every 32 row pairs, and at the end, all lanes finish theirs at once.
    int limit = my_sh;            // lane 0: uses that may be issued so far
    int n_pend = 0;
    float p_g = 0.0f, p_u = 0.0f;
    int p_h = 0;
    auto flush = [&]() {
        if (lane < n_pend) {
            const float hv = p_g / (1.0f + expf(-p_g)) * p_u;
            const __half hh = __float2half_rn(hv);
            if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(a.status, MOE_ERR_RANGE);
            a.h[p_h] = __half_as_ushort(hh);
        }
        n_pend = 0;
    };
    auto gate_up_use = [&](int q, float2 acc) {
        const int s = q % kFzStages;
        const int4 dsc = s_desc[warp][s];
        const float* scs = reinterpret_cast<const float*>(st_g(s) + 2 * gu_row);
        const float sg = scs[dsc.z], su = scs[dsc.w];
        __syncwarp();                                      // the stage is free again
        if (lane == 0)
            while (issued < limit && issued < q + 1 + kFzStages) issue(issued++);
        const float ag = warp_sum(acc.x), au = warp_sum(acc.y);
        if (lane == n_pend) {
            p_g = sg * (ag - off136);
            p_u = su * (au - off136);
            p_h = dsc.x * f + dsc.y;
        }
        if (++n_pend == kWarp) flush();
    };

    int q = 0;                    // next use to consume
    for (; ok && q < my_sh; ++q) {                         // the shared expert's row pairs
        if (lane == 0)
            while (issued < limit && issued < q + kFzStages) issue(issued++);
        if (!wait_use(q)) { ok = false; break; }
        gate_up_use(q, gu_dot(st_s(q % kFzStages), gu_row, lane, xp_s, nchunks));
    }

    // ---- B: selection by the whole CTA once every piece of the logits is stored.  The rings are
    //      idle: the router pieces, then the keys and logits, go to their start.
    __syncthreads();
    stamp(3);
    const uint32_t rbytes = ((uint32_t)n_units * 8u + 15u) & ~15u;
    uint2* keys = reinterpret_cast<uint2*>(rings + rbytes);    // keys, order-preserving integers
    double* lgs = reinterpret_cast<double*>(keys + E);
    if (tid == 0) {
        const bool bok = wait_arrivals(a.bar, s_base + (unsigned long long)G);
        if (bok) {
            bar_expect_tx(saddr(&s_rbar), rbytes);
            bulk_g2s(rings_s, a.rpart, rbytes, saddr(&s_rbar));
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
            const double* rp = reinterpret_cast<const double*>(rings);
            double l = 0.0;
            for (int p = 0; p < nch; ++p) l += rp[tid * nch + p];
            lgs[tid] = l;
            // key -> unsigned 64-bit integer of the same order (-0 folded into +0; NaN is -inf)
            const long long b = __double_as_longlong(topk_key(l, my_bias, a.router) + 0.0);
            const unsigned long long o = b < 0 ? ~(unsigned long long)b : (unsigned long long)b | (1ull << 63);
            keys[tid] = make_uint2((uint32_t)(o >> 32), (uint32_t)o);
        }
        sel = !__syncthreads_or(!landed);
        if (!sel && tid == 0) latch_status(a.status, MOE_ERR_TIMEOUT);
        stamp(5);
        // Selection in (key descending, index ascending) order, in two rounds.  Round 1: each warp
        // ranks its 32 experts among themselves; the k best of every warp are candidates (every
        // expert that beats one of the overall k best is itself among the overall k best, so the
        // overall k best are all candidates).  Round 2: each candidate's rank among the
        // candidates is its overall rank when that is below k.
        auto beats = [](uint2 kj, int j, uint2 ki, int i) {
            return (kj.x > ki.x) | ((kj.x == ki.x) & ((kj.y > ki.y) | ((kj.y == ki.y) & (j < i))));
        };
        const int nwe = (E + kWarp - 1) / kWarp;           // warps holding experts
        if (sel && warp < nwe) {
            const int e = tid;
            const uint2 mk = e < E ? keys[e] : make_uint2(0u, 0u);   // below every real key
            int rank = 0;
#pragma unroll 4
            for (int o = 1; o < kWarp; ++o) {
                const int jl = (lane + o) & (kWarp - 1);
                const uint2 kj = make_uint2(__shfl_sync(0xffffffffu, mk.x, jl), __shfl_sync(0xffffffffu, mk.y, jl));
                rank += beats(kj, warp * kWarp + jl, mk, e) ? 1 : 0;
            }
            if (lane < k) {
                cand_e[warp * k + lane] = -1;
                cand_k[warp * k + lane] = make_uint2(0u, 0u);
            }
            __syncwarp();
            if (e < E && rank < k) {
                cand_e[warp * k + rank] = e;
                cand_k[warp * k + rank] = mk;
            }
        }
        __syncthreads();
        stamp(12);
        const int nc = nwe * k;                            // candidate slots
        if (sel && tid < nc) {
            const int e = cand_e[tid];
            if (e >= 0) {
                const uint2 mk = cand_k[tid];
                int rank = 0;
#pragma unroll 8
                for (int c = 0; c < nc; ++c)               // empty slots hold key 0, below every real key
                    rank += beats(cand_k[c], cand_e[c], mk, e) ? 1 : 0;
                if (rank < k) {
                    sel_e[rank] = e;
                    sel_l[rank] = lgs[e];
                }
            }
        }
        __syncthreads();
        stamp(13);
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
    stamp(14);
    // the keys were written through the generic proxy; TMA writes into the same bytes come next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    stamp(15);
    __syncthreads();              // s_e, s_w set; the rings may be used again
    stamp(6);
    const bool routed = sel;

    // ---- C: the routed row pairs; then the first down stages (independent of h)
    for (int it = it0, row = it0 - (it0 / max(rj, 1)) * rj; it < it1; ++n_dn) {
        const int n = dn_count(it, row);
        it += n;
        row = row + n == rj ? 0 : row + n;
    }
    if (ok && routed) {
        limit = my_tasks + n_dn;
        for (; q < my_tasks; ++q) {
            if (lane == 0)
                while (issued < limit && issued < q + kFzStages) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            gate_up_use(q, gu_dot(st_s(q % kFzStages), gu_row, lane, xp_s, nchunks));
        }
        if (ok && lane == 0)
            while (issued < limit && issued < q + kFzStages) issue(issued++);
    }
    flush();

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
        float hs = 0.0f;                                   // sum of this slot's h
        int cu = it0 / max(rj, 1), crow = it0 - cu * rj, hu = -1;
        for (int it = it0; it < it1; ++q) {
            const int n = dn_count(it, crow);
            const float* scp = (cu < k ? a.dn_scale + (size_t)s_e[cu] * d : a.sh_dn_scale) + j0 + crow;
            const float my_sc = lane < n ? __ldg(scp + lane) : 0.0f;
            if (cu != hu) {                                // this slot's h (written by other CTAs)
                float hl = 0.0f;
#pragma unroll
                for (int j = 0; j < NCF; ++j) {
                    const int c = lane + kWarp * j;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint4 v = ld_cg16(a.h + (size_t)cu * f + (size_t)c * 32 + 8 * m);
                        pair_cols(v, &hr[j][4 * m]);
                        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
                            hl += hf.x + hf.y;
                        }
                    }
                }
                hs = warp_sum(hl);
                hu = cu;
            }
            if (lane == 0)
                while (issued < limit && issued < q + kFzStages) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            const uint32_t st = st_s(q % kFzStages);
#pragma unroll 1
            for (int rr = 0; rr < n; ++rr) {
                float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
                for (int j = 0; j < NCF; ++j) {
                    const uint4 wv = lds16(st + (uint32_t)rr * dn_row_b + (uint32_t)(lane + kWarp * j) * 16);
                    v0 = dot_word_f16top(wv.x, &hr[j][0], v0);
                    v1 = dot_word_f16top(wv.y, &hr[j][4], v1);
                    v0 = dot_word_f16top(wv.z, &hr[j][8], v0);
                    v1 = dot_word_f16top(wv.w, &hr[j][12], v1);
                }
                const float v = warp_sum(v0 + v1);         // sum (3/2 + s/16) h
                const float srow = __shfl_sync(0xffffffffu, my_sc, rr);
                if (lane == 0) ys[cu][crow + rr] = srow * fmaf(16.0f, v, -24.0f * hs);
            }
            __syncwarp();
            if (lane == 0)
                while (issued < limit && issued < q + 1 + kFzStages) issue(issued++);
            it += n;
            crow += n;
            if (crow == rj) {
                crow = 0;
                ++cu;
            }
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
    const int w = (int)((kSmemLimit - kStaticReserve - 2 * (size_t)L.d) / ((size_t)kFzStages * fz_stage_bytes(L)));
    return w > kFzMaxWarps ? kFzMaxWarps : w;
}
size_t fz_dyn_smem(const LayerDims& L) {
    return 2 * (size_t)L.d + (size_t)fz_warps(L) * kFzStages * fz_stage_bytes(L);
}
int fz_dn_rows(const LayerDims& L) {
    const int r = (int)(fz_stage_bytes(L) / (size_t)(L.f / 2));
    return r > kFzDnRowsMax ? kFzDnRowsMax : r;
}

const void* fz_pick(const LayerDims& L) {
    return L.f / 1024 == 1 ? (const void*)decode_fused_kernel<1> : (const void*)decode_fused_kernel<2>;
}

}  // namespace

bool decode_fused_shape_ok(const LayerDims& L) {
    if (!(L.wkind == MOE_W_INT4_ROWSCALE && L.d % 1024 == 0 && L.d / 1024 >= 1 && L.d / 1024 <= 8 &&
          (L.f == 1024 || L.f == 2048) && (!L.S || L.f_shared == L.f) && L.k + L.S <= kFzMaxSlots &&
          L.E <= kWarp * kFzMaxPer && L.k <= L.E && fz_warps(L) >= 4 && fz_dn_rows(L) >= 1))
        return false;
    // the selection keeps the router pieces, keys and logits in the (idle) rings; E <= threads
    const size_t dyn = (size_t)fz_warps(L) * kFzStages * fz_stage_bytes(L);   // the rings
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
    const size_t dyn = fz_dyn_smem(L);
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
    cfg.dynamicSmemBytes = fz_dyn_smem(L);
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
