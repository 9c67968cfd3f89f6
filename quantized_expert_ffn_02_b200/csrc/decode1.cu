// decode1.cu -- K4/K6 for a single token (T = 1) with int4 experts: the decode step of the layer.
//
// One token touches k routed experts plus the shared one; every weight byte is read once, so
// the step is bound by HBM.  Two kernels, chained with programmatic dependent launch (PDL):
//
//   gateup_t1   persistent, one CTA per SM.  Each lane keeps its share of the token's activations
//               in registers for the whole kernel (d/32 values, pre-paired to match the nibble
//               pairs).  Each warp streams its row pairs (a gate row and the matching up row) into
//               its own ring of shared-memory stages with TMA bulk copies, so the bytes in flight
//               do not cost registers; it reduces each pair with warp shuffles and writes h.  The
//               shared expert's rows need no routing and come first: they run while the router
//               kernel is still finishing, and `griddepcontrol.wait` is reached only before the
//               first routed row is fetched.
//   down_t1     one CTA per block of output rows, two warps per slot (routed experts in
//               ascending index, then the shared expert).  A warp keeps its slot's h in registers
//               and streams its rows through its own TMA ring; the weight copies start before
//               `griddepcontrol.wait` (they do not depend on h).  The CTA then adds the slots in
//               order with their gate weights (the combine), so y never goes through global memory.
//
// Dequantisation as in decode.cu: bf16 (136 + s) with the offset removed per row through the
// sum of x (computed here in fp64 from the registers); fp16 s exactly for the down rows.
//
// Data written by a kernel that may still run while this one runs (the router's tables, h) are
// read through L2 with ld.global.cg: the non-coherent path may return stale lines.
//
// Every wait on an mbarrier is bounded (about 2 s).  A warp that gives up latches
// MOE_ERR_TIMEOUT, waits (bounded again) for the copies it issued, and skips its remaining work.
#include "decode_common.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace qe {
namespace {

using namespace dec;

constexpr int kGuStages = 3;          // row pairs in flight per warp (gate/up)
constexpr int kGuMaxWarps = 12;
constexpr int kDnSlotWarps = 2;       // warps per slot (down)
constexpr int kDnRows = 4;            // rows per stage (down)
constexpr int kDnStages = 3;
constexpr int kDnMaxSlots = 10;       // k + 1
constexpr int kDnRowsMax = 64;        // output rows per CTA at most
constexpr size_t kSmemLimit = 227 * 1024;

// ---------------------------------------------------------------------------------------
// gate/up + SiLU, T = 1.  NCH = d / 1024 chunks of 32 columns per lane.
// Row pairs: [0, f_sh) of the shared expert (slot k), then u * f + r of routed expert ulist[u]
// (slot u: with one token the routed slots are the unique experts in ascending order).
// Warp gw takes tasks gw, gw + nw, ... (nw warps in the grid).
// ---------------------------------------------------------------------------------------
struct GuTask {
    const uint8_t* gate;     // gate row (the up row is fe rows further)
    const float* sc;         // scale of the gate row (the up row's is fe further)
    int r, fe, slot;
};

template <int NCH>
__global__ void __launch_bounds__(kGuMaxWarps * kWarp, 1)
gateup_t1_kernel(const uint8_t* __restrict__ gate_up, const float* __restrict__ gu_scale,
                 const uint8_t* __restrict__ sh_gate_up, const float* __restrict__ sh_gu_scale,
                 const uint16_t* __restrict__ x, int k, int d, int f, int f_sh, int S, const int32_t* ulist,
                 uint16_t* __restrict__ h, int fmax, int* status, const void* const* __restrict__ etab, int E) {
    // [warps][kGuStages][gate row | up row | 16 B holding the gate scale | 16 B holding the up scale]
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kGuMaxWarps][kGuStages];
    __shared__ int s_ulist[kGuMaxWarps][kDnMaxSlots];      // this warp's copy of the routed experts
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    const int nwarps_cta = blockDim.x / kWarp;
    const int gw = blockIdx.x * nwarps_cta + warp;
    const int nw = gridDim.x * nwarps_cta;
    const uint32_t rowbytes = (uint32_t)d / 2;
    const uint32_t stage_bytes = 2 * rowbytes + 32;
    const int n_shared_tasks = S ? f_sh : 0;
    const int n_tasks = n_shared_tasks + k * f;
    const int my_tasks = gw < n_tasks ? (n_tasks - gw + nw - 1) / nw : 0;
    const uint32_t ring = saddr(smem) + (uint32_t)warp * kGuStages * stage_bytes;
    const uint8_t* ring_g = smem + (size_t)warp * kGuStages * stage_bytes;
    if (lane == 0) {
        for (int s = 0; s < kGuStages; ++s) bar_init(saddr(&bars[warp][s]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    bool routed_ready = false;          // lane 0 only: the router kernel has finished
    auto task = [&](int i) {
        GuTask tk;
        const int t = gw + i * nw;
        if (t < n_shared_tasks) {
            tk.gate = sh_gate_up + (size_t)t * rowbytes;
            tk.sc = sh_gu_scale + t;
            tk.r = t;
            tk.fe = f_sh;
            tk.slot = k;
        } else {
            if (!routed_ready) {
                pdl_wait();
                pdl_trigger();          // the down kernel may now read the routing
                for (int q = 0; q < k; ++q) s_ulist[warp][q] = __ldcg(ulist + q);
                routed_ready = true;
            }
            const int t2 = t - n_shared_tasks;
            const int u = t2 / f, r = t2 % f;
            const int e = s_ulist[warp][u];
            tk.gate = ex_gate_up(etab, E, e) + (size_t)r * rowbytes;
            tk.sc = ex_gu_scale(etab, E, e) + r;
            tk.r = r;
            tk.fe = f;
            tk.slot = u;
        }
        return tk;
    };
    // lane 0 issues task i into stage i % kGuStages: both rows, and the 16-byte aligned slivers of
    // the scale arrays that hold their two scales (scale arrays are 16-byte aligned and a routed
    // expert's scales start at a multiple of 4 floats)
    auto sliver = [](const float* p) { return reinterpret_cast<const float*>((uintptr_t)p & ~(uintptr_t)15); };
    auto issue = [&](int i) {
        const GuTask tk = task(i);
        const uint32_t bar = saddr(&bars[warp][i % kGuStages]);
        const uint32_t dst = ring + (uint32_t)(i % kGuStages) * stage_bytes;
        bar_expect_tx(bar, stage_bytes);
        bulk_g2s(dst, tk.gate, rowbytes, bar);
        bulk_g2s(dst + rowbytes, tk.gate + (size_t)tk.fe * rowbytes, rowbytes, bar);
        bulk_g2s(dst + 2 * rowbytes, sliver(tk.sc), 16, bar);
        bulk_g2s(dst + 2 * rowbytes + 16, sliver(tk.sc + tk.fe), 16, bar);
    };
    int issued = 0;
    if (lane == 0)      // prologue: shared-expert rows only (they need no routing)
        while (issued < my_tasks && issued < kGuStages && gw + issued * nw < n_shared_tasks) issue(issued++);

    // the token's activations: lane owns chunks lane + 32 j
    // sum of x: each lane's share in fp32, the 32 partials in fp64 (the offset removed per row is
    // 136 times this sum; its error stays far below the rounding of the fp32 row sums)
    uint32_t xr[NCH][16];
    float xsl = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + kWarp * j;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint4 v = ld_ro16(x + (size_t)c * 32 + 8 * m);
            pair_cols(v, &xr[j][4 * m]);
            const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                xsl += __uint_as_float(ws[q] << 16) + __uint_as_float(ws[q] & 0xffff0000u);
        }
    }
    const double xs = warp_sum_d((double)xsl);
    const float off136 = 136.0f * (float)xs;

    bool ok = true;
    int i = 0;
    for (; i < my_tasks; ++i) {
        if (lane == 0 && issued == i) issue(issued++);         // a routed first task: fetch it now
        const int s = i % kGuStages;
        ok = bar_wait(saddr(&bars[warp][s]), (uint32_t)(i / kGuStages) & 1u);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t st = ring + (uint32_t)s * stage_bytes;
        float ag = 0.0f, au = 0.0f;
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
            const uint32_t off = (uint32_t)(lane + kWarp * j) * 16;
            const uint4 G = lds16(st + off), U = lds16(st + rowbytes + off);
            ag = dot_word_bf16(G.x, &xr[j][0], ag);
            au = dot_word_bf16(U.x, &xr[j][0], au);
            ag = dot_word_bf16(G.y, &xr[j][4], ag);
            au = dot_word_bf16(U.y, &xr[j][4], au);
            ag = dot_word_bf16(G.z, &xr[j][8], ag);
            au = dot_word_bf16(U.z, &xr[j][8], au);
            ag = dot_word_bf16(G.w, &xr[j][12], ag);
            au = dot_word_bf16(U.w, &xr[j][12], au);
        }
        // the row index and the two scales of this task, read before the stage is handed back
        const GuTask tk = task(i);
        const float* scs = reinterpret_cast<const float*>(ring_g + (size_t)s * stage_bytes + 2 * rowbytes);
        const float sg = scs[(uintptr_t)tk.sc / 4 & 3], su = scs[4 + ((uintptr_t)(tk.sc + tk.fe) / 4 & 3)];
        __syncwarp();                                          // stage s is free again
        if (lane == 0)
            while (issued < my_tasks && issued < i + 1 + kGuStages) issue(issued++);
        ag = warp_sum(ag);
        au = warp_sum(au);
        if (lane == 0) {
            const float gv = sg * (ag - off136);
            const float uv = su * (au - off136);
            const float hv = gv / (1.0f + expf(-gv)) * uv;
            const __half hh = __float2half_rn(hv);
            if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(status, MOE_ERR_RANGE);
            h[(size_t)tk.slot * fmax + tk.r] = __half_as_ushort(hh);
        }
    }
    if (lane == 0) {
        if (!ok) {
            latch_status(status, MOE_ERR_TIMEOUT);
            for (int j = i; j < issued; ++j)              // copies still in flight land before exit
                bar_wait(saddr(&bars[warp][j % kGuStages]), (uint32_t)(j / kGuStages) & 1u);
        }
        if (!routed_ready) {
            pdl_wait();
            pdl_trigger();
        }
    }
}

// ---------------------------------------------------------------------------------------
// down + combine, T = 1.  NCH = f / 1024 chunks of 32 K values per lane.
// CTA: output rows [j0, j0 + nj); warp w: slot u = w / 2 (u < k routed expert ulist[u], u == k the
// shared expert), half w % 2 of the CTA's rows, streamed kDnRows at a time.
// ---------------------------------------------------------------------------------------
template <int NCH>
__global__ void __launch_bounds__(kDnMaxSlots * kDnSlotWarps * kWarp, 1)
down_t1_kernel(const uint8_t* __restrict__ down, const float* __restrict__ dn_scale,
               const uint8_t* __restrict__ sh_down, const float* __restrict__ sh_dn_scale, const uint16_t* h,
               int fmax, int k, int d, int f, int S, const int32_t* ulist, const float* wts, const int32_t* asc,
               void* __restrict__ out, int out_bf16, int rj, int* status, const void* const* __restrict__ etab,
               int E) {
    extern __shared__ __align__(128) uint8_t smem[];          // [warps][kDnStages][kDnRows * rowbytes]
    __shared__ __align__(8) uint64_t bars[kDnMaxSlots * kDnSlotWarps][kDnStages];
    __shared__ float ys[kDnMaxSlots][kDnRowsMax];
    __shared__ float gate_w[kDnMaxSlots];
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    const int u = warp / kDnSlotWarps, half = warp % kDnSlotWarps;
    const int j0 = blockIdx.x * rj;
    const int nj = max(0, min(rj, d - j0));
    // this warp's rows: [r0, r1) of the CTA's block
    const int per = (nj + kDnSlotWarps - 1) / kDnSlotWarps;
    const int r0 = min(nj, half * per), r1 = min(nj, r0 + per);
    const int nrows = r1 - r0;
    const int nstages = (nrows + kDnRows - 1) / kDnRows;
    const bool shared = u == k;
    const uint32_t rowbytes = (uint32_t)f / 2;
    const uint32_t stage_bytes = kDnRows * rowbytes;
    const uint32_t ring = saddr(smem) + (uint32_t)warp * kDnStages * stage_bytes;
    // routing is final when this grid starts (the gate/up kernel triggered after its own wait)
    const int e = shared ? -1 : __ldcg(ulist + u);
    const uint8_t* W = shared ? sh_down : ex_down(etab, E, e);
    const float* sc = shared ? sh_dn_scale : ex_dn_scale(etab, E, e);
    if (u < k && half == 0 && lane == 0) gate_w[u] = __ldcg(wts + __ldcg(asc + u));
    if (lane == 0) {
        for (int s = 0; s < kDnStages; ++s) bar_init(saddr(&bars[warp][s]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    auto issue = [&](int g) {       // stage g: rows r0 + 4g .. (contiguous)
        const int a = r0 + g * kDnRows, n = min(kDnRows, r1 - a);
        const uint32_t bar = saddr(&bars[warp][g % kDnStages]);
        bar_expect_tx(bar, (uint32_t)n * rowbytes);
        bulk_g2s(ring + (uint32_t)(g % kDnStages) * stage_bytes, W + (size_t)(j0 + a) * rowbytes,
                 (uint32_t)n * rowbytes, bar);
    };
    int issued = 0;
    if (lane == 0)                  // the weights do not depend on h: start before the wait
        while (issued < nstages && issued < kDnStages) issue(issued++);
    // lane q holds the scale of this warp's row q (a warp has at most 32 rows)
    const float my_sc = lane < nrows ? __ldg(sc + j0 + r0 + lane) : 0.0f;
    pdl_wait();                     // h is complete
    uint32_t hr[NCH][16];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + kWarp * j;
#pragma unroll
        for (int m = 0; m < 4; ++m) pair_cols(ld_cg16(h + (size_t)u * fmax + (size_t)c * 32 + 8 * m), &hr[j][4 * m]);
    }
    bool ok = true;
    int g = 0;
    for (; g < nstages; ++g) {
        const int s = g % kDnStages;
        ok = bar_wait(saddr(&bars[warp][s]), (uint32_t)(g / kDnStages) & 1u);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t st = ring + (uint32_t)s * stage_bytes;
        const int a = r0 + g * kDnRows, n = min(kDnRows, r1 - a);
        float acc[kDnRows];
#pragma unroll
        for (int q = 0; q < kDnRows; ++q) {
            float v = 0.0f;
            if (q < n) {
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
                    const uint4 wv = lds16(st + (uint32_t)q * rowbytes + (uint32_t)(lane + kWarp * j) * 16);
                    v = dot_word_f16(wv.x, &hr[j][0], v);
                    v = dot_word_f16(wv.y, &hr[j][4], v);
                    v = dot_word_f16(wv.z, &hr[j][8], v);
                    v = dot_word_f16(wv.w, &hr[j][12], v);
                }
            }
            acc[q] = v;
        }
        __syncwarp();
        if (lane == 0 && issued < nstages) issue(issued++);
#pragma unroll
        for (int q = 0; q < kDnRows; ++q) {
            const float v = warp_sum(acc[q]);
            const float s_row = __shfl_sync(0xffffffffu, my_sc, (a - r0 + q) & 31);
            if (lane == 0 && q < n) ys[u][a + q] = s_row * v;
        }
    }
    if (lane == 0 && !ok) {
        latch_status(status, MOE_ERR_TIMEOUT);
        for (int j = g; j < issued; ++j) bar_wait(saddr(&bars[warp][j % kDnStages]), (uint32_t)(j / kDnStages) & 1u);
    }
    __syncthreads();
    // combine: routed slots in ascending expert order, then the shared expert
    for (int i = threadIdx.x; i < nj; i += blockDim.x) {
        float o = 0.0f;
        for (int s = 0; s < k; ++s) o = fmaf(gate_w[s], ys[s][i], o);
        if (S) o += ys[k][i];
        if (out_bf16)
            static_cast<__nv_bfloat16*>(out)[j0 + i] = __float2bfloat16_rn(o);
        else
            static_cast<float*>(out)[j0 + i] = o;
    }
}

size_t gu_stage_bytes(const LayerDims& L) { return (size_t)L.d + 32; }   // two rows of d/2 bytes + scales
int gu_warps(const LayerDims& L) {
    const size_t per_warp = (size_t)kGuStages * gu_stage_bytes(L);
    const int w = (int)((kSmemLimit - 4096) / per_warp);
    return w > kGuMaxWarps ? kGuMaxWarps : w;
}
size_t dn_smem(const LayerDims& L) {
    return (size_t)(L.k + L.S) * kDnSlotWarps * kDnStages * kDnRows * (L.f / 2);
}

}  // namespace

bool decode_t1_supported(const LayerDims& L) {
    return L.wkind == MOE_W_INT4_ROWSCALE && L.d % 1024 == 0 && L.d / 1024 <= 8 && L.f % 1024 == 0 &&
           L.f / 1024 <= 4 && (!L.S || L.f_shared == L.f) && L.k + L.S <= kDnMaxSlots && gu_warps(L) >= 4 &&
           dn_smem(L) <= kSmemLimit - 4096;  // 4 KB left for static shared memory
}

cudaError_t prepare_decode(const LayerDims& L) {
    if (!decode_t1_supported(L)) return cudaSuccess;
    // opt each kernel into all the dynamic shared memory its static part leaves free
    cudaError_t e = cudaSuccess;
    auto opt_in = [](const void* fn) {
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, fn);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)(kSmemLimit - fa.sharedSizeBytes));
    };
#define QE_ATTR(KERN) \
    if (e == cudaSuccess) e = opt_in((const void*)KERN);
    QE_ATTR(gateup_t1_kernel<1>) QE_ATTR(gateup_t1_kernel<2>) QE_ATTR(gateup_t1_kernel<3>) QE_ATTR(gateup_t1_kernel<4>)
    QE_ATTR(gateup_t1_kernel<5>) QE_ATTR(gateup_t1_kernel<6>) QE_ATTR(gateup_t1_kernel<7>) QE_ATTR(gateup_t1_kernel<8>)
    QE_ATTR(down_t1_kernel<1>) QE_ATTR(down_t1_kernel<2>) QE_ATTR(down_t1_kernel<3>) QE_ATTR(down_t1_kernel<4>)
#undef QE_ATTR
    return e;
}

cudaError_t launch_decode_t1(const LayerDims& L, const moe_weights& W, const uint16_t* x, const Workspace& ws,
                             void* out, int num_sms, const Launch& ctx) {
    const int fmax = L.f;
    const int nchx = L.d / 1024, nchf = L.f / 1024;
    const int guw = gu_warps(L);
    const size_t gu_smem = (size_t)guw * kGuStages * gu_stage_bytes(L);
    cudaError_t e = cudaSuccess;
    prof_mark(ctx.prof, MOE_KERNEL_GATEUP, true, ctx.s);
#define QE_GU(N)                                                                                                      \
    case N:                                                                                                           \
        e = launch_pdl(L.pdl != 0, gateup_t1_kernel<N>, dim3(num_sms), dim3(guw * kWarp), gu_smem, ctx.s,              \
                       (const uint8_t*)W.gate_up, W.gate_up_scale, (const uint8_t*)W.shared_gate_up,                  \
                       W.shared_gate_up_scale, x, L.k, L.d, L.f, L.f_shared, L.S, (const int32_t*)ws.ulist, ws.h,     \
                       fmax, ws.status, (const void* const*)ws.etab, L.E);                                            \
        break;
    switch (nchx) {
        QE_GU(1) QE_GU(2) QE_GU(3) QE_GU(4) QE_GU(5) QE_GU(6) QE_GU(7) QE_GU(8)
        default: return cudaErrorInvalidValue;
    }
#undef QE_GU
    prof_mark(ctx.prof, MOE_KERNEL_GATEUP, false, ctx.s);
    if (e != cudaSuccess) return e;
    ++*ctx.launches;
    int rj = (L.d + num_sms - 1) / num_sms;
    if (rj > kDnRowsMax) rj = kDnRowsMax;
    const unsigned grid = (unsigned)((L.d + rj - 1) / rj);
    const unsigned threads = (unsigned)(L.k + L.S) * kDnSlotWarps * kWarp;
    const size_t dsm = dn_smem(L);
    prof_mark(ctx.prof, MOE_KERNEL_DOWN, true, ctx.s);
#define QE_DN(N)                                                                                                      \
    case N:                                                                                                           \
        e = launch_pdl(L.pdl != 0, down_t1_kernel<N>, dim3(grid), dim3(threads), dsm, ctx.s, (const uint8_t*)W.down,   \
                       W.down_scale, (const uint8_t*)W.shared_down, W.shared_down_scale, (const uint16_t*)ws.h, fmax, \
                       L.k, L.d, L.f, L.S, (const int32_t*)ws.ulist, (const float*)ws.wts, (const int32_t*)ws.asc,    \
                       out, L.out_bf16, rj, ws.status, (const void* const*)ws.etab, L.E);                             \
        break;
    switch (nchf) {
        QE_DN(1) QE_DN(2) QE_DN(3) QE_DN(4)
        default: return cudaErrorInvalidValue;
    }
#undef QE_DN
    prof_mark(ctx.prof, MOE_KERNEL_DOWN, false, ctx.s);
    if (e != cudaSuccess) return e;
    ++*ctx.launches;
    return cudaSuccess;
}

}  // namespace qe
