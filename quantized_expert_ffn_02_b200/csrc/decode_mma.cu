// decode_mma.cu -- K4 for small batches (T >= 2) with int4 experts: the batch-union expert FFN as
// tensor-core products of 16 weight rows by 8 tokens (or slots).
//
// The colibri README ("The idea"; "What's implemented": batch-union MoE) reads each chosen
// expert once per call and applies it to every token routed to it.  Here each chosen expert's
// tokens form groups of at most 8 ("columns"), and one mma.sync m16n8k16 multiplies 16 weight
// rows by a group: D[row][col] = sum_k W[row][k] * v[col][k], with the int4 codes decoded in
// registers and the K dimension reduced inside the instruction, so a row's dot products need no
// reduction across lanes.
//
//   gate/up (GU): the 16 rows are 8 gate rows and the matching 8 up rows, so lane (g, c) of the
//     warp ends with gate and up of row g for columns 2c and 2c + 1 and applies SiLU at once;
//     v = x~ = x 2^sigma (fp16, one power of two per token), h goes to HBM as fp16.
//   down (DN): 16 down rows against v = h~ = h 2^tau per slot; y goes to HBM per slot (fp32) and
//     the combine kernel adds the slots.
//
// Work: a unit is one group of up to 8 columns of one chosen expert (or of the shared expert),
// and its rows form 16-row blocks.  The blocks of all units are laid end to end and every CTA
// takes one contiguous range of them, so the CTAs get equal shares and a CTA meets only one or
// two units: it brings a unit's v rows into shared memory once, all its warps convert them, and
// the warps split the unit's blocks of the range.  Each warp streams its blocks' rows through a
// private ring of TMA bulk copies (16 rows x 512 bytes per stage), issued ahead across blocks
// and units, so HBM keeps streaming while the CTA converts the next unit's v.
//
// Decoding (as in the single-launch kernel): a code s is stored as the nibble n, n ^ 8 = s + 8.
// One LOP3 puts the nibble pair (i, i+4) of a word at fp16 mantissa bits 0..3 -- the exact value
// (s + 8) 2^-24 -- or, for the pair (i + 1, i + 5), at bits 4..7 -- (s + 8) 2^-20, met by v values
// stored x 2^-4; so every product is (s + 8) v~ 2^-24 exactly, and sum s v~ = 2^24 D - 8 sum v~.
// K order: word m of a lane's 16 bytes holds 8 columns; its MMA pair takes columns (0, 4) and
// (1, 5), then (2, 6) and (3, 7): the same order on both operands.
#include "decode_common.cuh"

#include <cuda_fp16.h>

namespace qe {
namespace {

using namespace dec;

constexpr int kUMaxWarps = 12;                // (the register budget allows 8 accumulators)
constexpr int kUStages = 2;                 // ring stages per warp
// Bytes of a weight row per stage: 256 (512 codes) for gate/up, 512 for down.  Gate/up holds
// its 8 columns of x (2d bytes each) beside the rings, so smaller stages buy more warps (12
// instead of 6 for d = 6144: gate/up 437 -> 383 us at T = 32); down's h columns are small and it
// already runs 10 warps, where 256-byte stages measured slower (178 -> 195 us).
template <bool GU> constexpr int u_chunk() { return GU ? 256 : 512; }
template <bool GU> constexpr int u_steps() { return u_chunk<GU>() / 64; }   // MMA steps (128 codes) per stage
// Shared-memory bytes per row in a stage: the lanes of rows g and g + 1 then meet different
// banks (the pitch is 16 words past a multiple of 32 words for both chunk sizes).
template <bool GU> constexpr int u_pitch() { return u_chunk<GU>() + 64; }
template <bool GU> constexpr int u_stage() { return 16 * u_pitch<GU>(); }
constexpr int kUCols = 8;                   // columns (tokens or slots) per unit
constexpr int kUChains = 8;                 // independent accumulators per warp
constexpr size_t kUSmemLimit = 227 * 1024;
constexpr int kUStaticReserve = 8192;       // static shared memory, rounded up
constexpr int kUMaxUnique = 1024;

struct UArgs {
    const void* const* etab;   // [4][E] the layer's per-expert pointers
    int E;
    const uint8_t* sh_w;       // the shared expert's gate/up (GU) or down (DN) rows
    const float* sh_sc;        // and their scales
    const int32_t* ulist;      // chosen experts, ascending
    const int32_t* n_unique;
    const int32_t* cnt;        // tokens per expert
    const int32_t* off;        // first slot per expert
    const int32_t* perm;       // slot -> t * k + rank
    int T, k, S, d, f, f_sh;
    const uint16_t* src;       // GU: x [T][d] bf16; DN: h [slots][src_ld] fp16
    int src_ld;
    void* dst;                 // GU: h [slots][dst_ld] fp16; DN: y [slots][dst_ld] fp32
    int dst_ld;
    int vrows;                 // rows of the v region (columns per unit, at most kUCols)
    int* status;
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) { return lop_sel_xor(w, 0x000F000Fu, 0x00080008u); }
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) { return lop_sel_xor(w, 0x00F000F0u, 0x00800080u); }
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }
__device__ __forceinline__ int scale_exp(float vmax) {
    if (!(vmax > 0.0f) || !isfinite(vmax)) return 0;
    const int e = (int)((__float_as_uint(vmax) >> 23) & 0xff) - 127;
    return max(-100, min(100, 14 - e));
}
// Position of 8-column group q in a v row: within each 16 groups, the second 8 have their pairs
// (q, q ^ 2) exchanged, so the 8 lanes of a shared-memory phase read 8 different bank quads.
__device__ __forceinline__ int vpos(int q) { return q ^ (((q >> 3) & 1) << 1); }

// 8 values (bf16 or fp16 bits) of one group -> the four fp16 operand pairs (0,4), (1,5)/16,
// (2,6), (3,7)/16 scaled by 2^e; adds the scaled values (unscaled positions) to sum.
template <bool BF16>
__device__ __forceinline__ uint4 to_pairs(uint4 v, float s, float s16, float& sum) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float c[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (BF16) {
            c[2 * i] = __uint_as_float(w[i] << 16);
            c[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        } else {
            const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            c[2 * i] = p.x;
            c[2 * i + 1] = p.y;
        }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float m = (i & 1) ? s16 : s;
        const __half2 r = __floats2half2_rn(c[i] * m, c[i + 4] * m);
        o[i] = *reinterpret_cast<const uint32_t*>(&r);
        const float2 b = __half22float2(r);
        sum += (i & 1) ? 16.0f * (b.x + b.y) : (b.x + b.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// A unit: which expert, which of its columns, and its blocks.
struct Unit {
    int u;          // unit number (routed units first, then the shared expert's)
    int e;          // expert, or -1 for the shared expert
    int j0, n;      // first member of the bucket and the number of columns (1..8)
    int K;          // reduction length (codes per row)
    int first;      // the unit's first block in the global block order
    int nb;         // 16-row blocks of the unit
};

template <bool GU>
__global__ void __launch_bounds__(kUMaxWarps * kWarp, 1) union_mma_kernel(const UArgs a) {
    // Launched with programmatic dependent launch after the previous kernel of the layer: wait
    // for its results before reading anything, then let the next kernel launch.
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kUMaxWarps][kUStages];
    __shared__ __align__(8) uint64_t vbar;                 // a unit's v rows landed
    __shared__ int s_pre[kUMaxUnique + 1];                 // units before chosen expert i
    __shared__ int s_col_slot[kUCols], s_col_tok[kUCols];
    __shared__ int s_sig[kUCols];
    __shared__ float s_vsum[kUCols];
    __shared__ float s_pmax[kUCols][kUMaxWarps];           // per row, per converting warp
    __shared__ double s_psum[kUCols][kUMaxWarps];
    __shared__ int s_abort;
    __shared__ int s_blk[2];                               // this CTA's block range

    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int nwc = blockDim.x / kWarp;
    const int G = gridDim.x;
    const int g = lane >> 2, c = lane & 3;
    const int Kmax = GU ? a.d : max(a.f, a.S ? a.f_sh : 0);
    const uint32_t vrs = (uint32_t)Kmax * 2u + 16u;       // v row pitch (bytes)
    const uint32_t v_s = saddr(smem);
    const uint32_t rings_s = v_s + (uint32_t)a.vrows * vrs;
    constexpr int kUChunk = u_chunk<GU>(), kUSteps = u_steps<GU>(), kURowPitch = u_pitch<GU>(), kUStage = u_stage<GU>();
    const uint32_t ring_s = rings_s + (uint32_t)warp * kUStages * kUStage;
    const int nu = *a.n_unique;
    const int nb_r = GU ? a.f / 8 : a.d / 16;              // blocks of a routed unit
    const int nb_s = GU ? a.f_sh / 8 : a.d / 16;           // of a shared-expert unit

    // ---- prologue: units per chosen expert (groups of kUCols columns), their prefix, and this
    //      CTA's share of the blocks
    if (tid == 0) {
        for (int s = 0; s < kUMaxWarps; ++s)
            for (int q = 0; q < kUStages; ++q) bar_init(saddr(&bars[s][q]), 1);
        bar_init(saddr(&vbar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
    }
    for (int i = tid; i < nu; i += blockDim.x) s_pre[i + 1] = (a.cnt[a.ulist[i]] + kUCols - 1) / kUCols;
    if (tid == 0) s_pre[0] = 0;
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < nu; ++i) s_pre[i + 1] += s_pre[i];
        const int64_t nb = (int64_t)s_pre[nu] * nb_r + (a.S ? (int64_t)((a.T + kUCols - 1) / kUCols) * nb_s : 0);
        s_blk[0] = (int)(nb * blockIdx.x / G);
        s_blk[1] = (int)(nb * (blockIdx.x + 1) / G);
    }
    __syncthreads();
    const int n_routed_units = s_pre[nu];
    const int blk_end = s_blk[1];

    // the unit that holds global block i
    auto unit_at = [&](int i) -> Unit {
        Unit un;
        const int routed_blocks = n_routed_units * nb_r;
        if (i < routed_blocks) {
            un.u = i / nb_r;
            int lo = 0, hi = nu - 1;                       // chosen expert with s_pre[lo] <= u < s_pre[lo + 1]
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_pre[mid] <= un.u) lo = mid; else hi = mid - 1;
            }
            un.e = a.ulist[lo];
            un.j0 = (un.u - s_pre[lo]) * kUCols;
            un.n = min(kUCols, a.cnt[un.e] - un.j0);
            un.K = GU ? a.d : a.f;
            un.first = un.u * nb_r;
            un.nb = nb_r;
        } else {
            const int us = (i - routed_blocks) / nb_s;
            un.u = n_routed_units + us;
            un.e = -1;
            un.j0 = us * kUCols;
            un.n = min(kUCols, a.T - un.j0);
            un.K = GU ? a.d : a.f_sh;
            un.first = routed_blocks + us * nb_s;
            un.nb = nb_s;
        }
        return un;
    };
    auto rows_of = [&](int e, const float*& sc) -> const uint8_t* {
        if (e < 0) {
            sc = a.sh_sc;
            return a.sh_w;
        }
        sc = GU ? ex_gu_scale(a.etab, a.E, e) : ex_dn_scale(a.etab, a.E, e);
        return GU ? ex_gate_up(a.etab, a.E, e) : ex_down(a.etab, a.E, e);
    };

    // ---- the warp's use stream: the segments of the CTA's range (a segment: the range's blocks
    //      of one unit), in each the warp's blocks seg_lo + warp + j nwc, in each block its K
    //      chunks.  The issuer (lanes 0 .. 15 copy one row each) runs up to kUStages uses ahead of
    //      the consumer, across blocks and segments.
    struct Cursor {
        int seg_hi;            // end of the current segment (global block index); -1: done
        int b;                 // current global block
        int kc, nkc;           // K chunk, chunks per row
        int first, fe;         // the unit's first block; gate/up: offset of the up rows
        const uint8_t* W;
        size_t rowb;           // bytes per weight row
    };
    auto cursor_seg = [&](Cursor& cu, int i) {
        if (i >= blk_end) {
            cu.seg_hi = -1;
            return;
        }
        const Unit un = unit_at(i);
        cu.seg_hi = min(blk_end, un.first + un.nb);
        cu.b = i + warp;
        cu.kc = 0;
        cu.nkc = un.K / (2 * kUChunk);
        cu.first = un.first;
        cu.fe = un.e < 0 ? a.f_sh : a.f;
        const float* sc;
        cu.W = rows_of(un.e, sc);
        cu.rowb = (size_t)un.K / 2;
    };
    auto cursor_settle = [&](Cursor& cu) {
        while (cu.seg_hi >= 0 && cu.b >= cu.seg_hi) cursor_seg(cu, cu.seg_hi);
    };
    Cursor is;
    cursor_seg(is, s_blk[0]);
    cursor_settle(is);
    int issued = 0, used = 0;
    auto issue_one = [&]() {  // whole warp: lane 0 arms the barrier, lanes 0..15 copy one row each
        const int s = issued % kUStages;
        const uint32_t bar = saddr(&bars[warp][s]);
        if (lane == 0) bar_expect_tx(bar, 16u * kUChunk);
        __syncwarp();
        if (lane < 16) {
            const int lb = is.b - is.first;                // block within the unit
            size_t row;
            if (GU) row = lane < 8 ? (size_t)lb * 8 + lane : (size_t)is.fe + (size_t)lb * 8 + (lane - 8);
            else row = (size_t)lb * 16 + lane;
            bulk_g2s(ring_s + (uint32_t)s * kUStage + (uint32_t)lane * kURowPitch,
                     is.W + row * is.rowb + (size_t)is.kc * kUChunk, kUChunk, bar);
        }
        ++issued;
        if (++is.kc == is.nkc) {
            is.kc = 0;
            is.b += nwc;
            cursor_settle(is);
        }
    };
    // the CTA's abort flag, read once by lane 0 for the whole warp (so the warp stays converged)
    auto aborted = [&]() { return __shfl_sync(0xffffffffu, *(volatile int*)&s_abort, 0) != 0; };
    auto top_up = [&]() {
        if (aborted()) return;
        while (is.seg_hi >= 0 && issued < used + kUStages) issue_one();
    };
    top_up();

    int vphase = 0;
    for (int i = s_blk[0]; i < blk_end;) {
        const Unit un = unit_at(i);
        const int seg_hi = min(blk_end, un.first + un.nb);
        // ---- the unit's columns: v rows into shared memory, converted in place by all warps
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the last unit's conversion writes
        __syncthreads();                                   // every warp is done with the last unit's v
        if (tid < un.n) {
            const int j = un.j0 + tid;
            int tok, slot;
            if (un.e < 0) {
                tok = j;
                slot = a.T * a.k + j;
            } else {
                slot = a.off[un.e] + j;
                tok = a.perm[slot] / a.k;
            }
            s_col_slot[tid] = slot;
            s_col_tok[tid] = tok;
        }
        __syncthreads();
        const uint32_t vbytes = (uint32_t)un.K * 2u;
        if (tid == 0) {
            bar_expect_tx(saddr(&vbar), (uint32_t)un.n * vbytes);
            for (int j = 0; j < un.n; ++j) {
                const uint16_t* srow = a.src + (size_t)(GU ? s_col_tok[j] : s_col_slot[j]) * a.src_ld;
                bulk_g2s(v_s + (uint32_t)j * vrs, srow, vbytes, saddr(&vbar));
            }
        }
        const bool vok = bar_wait(saddr(&vbar), (uint32_t)(vphase & 1));
        ++vphase;
        if (!vok && lane == 0) {
            latch_status(a.status, MOE_ERR_TIMEOUT);
            s_abort = 1;
        }
        // worker (row j, part s): S parts per row when the rows are no more than the warps
        const int ngr = un.K / 8;                          // 8-column groups per row
        const int S = un.n <= nwc ? nwc / un.n : 1;
        const int wj = un.n <= nwc ? warp % un.n : warp, ws = un.n <= nwc ? warp / un.n : 0;
        const int wjstep = un.n <= nwc ? un.n : nwc;
        const bool worker = ws < S;
        if (worker)
            for (int j = wj; j < un.n; j += (un.n <= nwc ? un.n + nwc : wjstep)) {   // one row when n <= warps
                const uint32_t row = v_s + (uint32_t)j * vrs;
                float m = 0.0f;
                for (int q = ws * kWarp + lane; q < ngr; q += kWarp * S) {
                    const uint4 v = lds16(row + 16u * q);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        float lo, hi;
                        if (GU) {
                            lo = __uint_as_float(w[t] << 16);
                            hi = __uint_as_float(w[t] & 0xffff0000u);
                        } else {
                            const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[t]));
                            lo = p.x;
                            hi = p.y;
                        }
                        m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) s_pmax[j][ws] = m;
            }
        __syncthreads();
        if (tid < un.n) {
            float m = 0.0f;
            for (int s = 0; s < S; ++s) m = fmaxf(m, s_pmax[tid][s]);
            s_sig[tid] = scale_exp(m);
        }
        __syncthreads();
        if (worker)
            for (int j = wj; j < un.n; j += (un.n <= nwc ? un.n + nwc : wjstep)) {
                const uint32_t row = v_s + (uint32_t)j * vrs;
                const int sig = s_sig[j];
                const float s1 = exp2i(sig), s16 = exp2i(sig - 4);
                float part = 0.0f;
                // in place: groups with bit 3 clear stay; with bit 3 set, q and q ^ 2 trade places
                // (the lane that holds the one with bit 1 clear moves both)
                for (int q = ws * kWarp + lane; q < ngr; q += kWarp * S) {
                    if ((q >> 3) & 1) {
                        if ((q >> 1) & 1) continue;
                        const uint4 v0 = lds16(row + 16u * q), v1 = lds16(row + 16u * (q ^ 2));
                        const uint4 p0 = to_pairs<GU>(v0, s1, s16, part), p1 = to_pairs<GU>(v1, s1, s16, part);
                        sts16(row + 16u * (q ^ 2), p0);
                        sts16(row + 16u * q, p1);
                    } else {
                        sts16(row + 16u * q, to_pairs<GU>(lds16(row + 16u * q), s1, s16, part));
                    }
                }
                const double ps = warp_sum_d((double)part);
                if (lane == 0) s_psum[j][ws] = ps;
            }
        __syncthreads();
        if (tid < un.n) {
            double t = 0.0;
            for (int s = 0; s < S; ++s) t += s_psum[tid][s];
            s_vsum[tid] = (float)t;
        }
        __syncthreads();

        // ---- this warp's blocks of the segment
        const float* sc;
        rows_of(un.e, sc);
        const int nkc = un.K / (2 * kUChunk);
        const int fe = un.e < 0 ? a.f_sh : a.f;
        const uint32_t vrow = v_s + (uint32_t)g * vrs;     // column g's v row (rows >= n hold junk; unused)
        // lane constants: its A bytes in a stage row, and its four v groups of a step (group
        // 4c + m sits at 4c + (m ^ 2) when c >= 2, the second 8 of each 16; see vpos)
        const uint32_t ao0 = (uint32_t)g * kURowPitch + 16u * c, ao1 = ao0 + 8u * kURowPitch;
        const uint32_t xsw = c >= 2 ? 2u : 0u;
        for (int b = i + warp; b < seg_hi; b += nwc) {
            const int lb = b - un.first;
            float acc[kUChains][4] = {};
            for (int kc = 0; kc < nkc; ++kc) {
                bool ok = !aborted();
                if (ok) {
                    ok = bar_wait(saddr(&bars[warp][used % kUStages]), (uint32_t)((used / kUStages) & 1));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok && lane == 0) {
                        latch_status(a.status, MOE_ERR_TIMEOUT);
                        s_abort = 1;
                    }
                }
                if (ok) {
                    const uint32_t st = ring_s + (uint32_t)(used % kUStages) * kUStage;
                    const uint32_t xb = vrow + 16u * (uint32_t)(kc * (2 * kUChunk / 8) + 4 * c);
#pragma unroll
                    for (int s = 0; s < kUSteps; ++s) {    // 128 codes per step
                        const uint4 A0 = lds16(st + ao0 + (uint32_t)(s * 64));
                        const uint4 A1 = lds16(st + ao1 + (uint32_t)(s * 64));
                        const uint32_t w0[4] = {A0.x, A0.y, A0.z, A0.w}, w1[4] = {A1.x, A1.y, A1.z, A1.w};
                        uint4 X[4];
#pragma unroll
                        for (int m = 0; m < 4; ++m) X[m] = lds16(xb + (uint32_t)(s * 256) + 16u * ((uint32_t)m ^ xsw));
                        // columns (0, 4) and (1, 5) of the four words into accumulators 0..3,
                        // (2, 6) and (3, 7) into 4..7: eight independent chains
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            mma16816(acc[m], nib_lo(w0[m]), nib_lo(w1[m]), nib_hi(w0[m]), nib_hi(w1[m]), X[m].x, X[m].y);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const uint32_t u0 = w0[m] >> 8, u1 = w1[m] >> 8;
                            mma16816(acc[4 + m], nib_lo(u0), nib_lo(u1), nib_hi(u0), nib_hi(u1), X[m].z, X[m].w);
                        }
                    }
                }
                __syncwarp();                              // the stage is free again
                ++used;
                top_up();
            }
            if (aborted()) continue;
            // ---- epilogue: lane (g, c) holds rows g and g + 8 for columns 2c and 2c + 1
            float d4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                d4[t] = ((acc[0][t] + acc[1][t]) + (acc[2][t] + acc[3][t])) + ((acc[4][t] + acc[5][t]) + (acc[6][t] + acc[7][t]));
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int col = 2 * c + h2;
                if (col >= un.n) continue;
                const float un_s = exp2i(-s_sig[col]);
                const float vs = 8.0f * s_vsum[col];
                const float lo = fmaf(d4[h2], 16777216.0f, -vs) * un_s;        // sum s v over row g (or 8 + g)
                const float hi = fmaf(d4[2 + h2], 16777216.0f, -vs) * un_s;
                const int slot = s_col_slot[col];
                if (GU) {
                    const int r = lb * 8 + g;                                   // row pair within the unit
                    const float gt = __ldg(sc + r) * lo, up = __ldg(sc + fe + r) * hi;
                    const float hv = gt / (1.0f + expf(-gt)) * up;
                    const __half hh = __float2half_rn(hv);
                    if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(a.status, MOE_ERR_RANGE);
                    static_cast<uint16_t*>(a.dst)[(size_t)slot * a.dst_ld + r] = __half_as_ushort(hh);
                } else {
                    const int j0 = lb * 16 + g;
                    float* y = static_cast<float*>(a.dst) + (size_t)slot * a.dst_ld;
                    y[j0] = __ldg(sc + j0) * lo;
                    y[j0 + 8] = __ldg(sc + j0 + 8) * hi;
                }
            }
        }
        i = seg_hi;
    }
    // copies still in flight (only after an abort: then uses may have been passed unwaited) land
    // before the CTA's shared memory goes away; only the last use of each stage can be in flight
    if (lane == 0)
        for (int q = max(0, issued - kUStages); q < issued; ++q)
            bar_wait(saddr(&bars[warp][q % kUStages]), (uint32_t)((q / kUStages) & 1));
    __syncwarp();
}

int union_warps(size_t vbytes, int stage) {
    const size_t room = kUSmemLimit - kUStaticReserve - vbytes;
    const int w = (int)(room / ((size_t)kUStages * stage));
    return w > kUMaxWarps ? kUMaxWarps : w;
}

}  // namespace

bool decode_mma_ok(const LayerDims& L, int T) {
    if (L.wkind != MOE_W_INT4_ROWSCALE || T < 2) return false;
    if (L.d % 1024 || L.f % 1024 || (L.S && L.f_shared % 1024)) return false;
    if (L.E > kUMaxUnique) return false;
    const int vrows = T < kUCols ? T : kUCols;
    const size_t gu_v = (size_t)vrows * (2 * (size_t)L.d + 16);
    const size_t dn_v = (size_t)vrows * (2 * (size_t)(L.S && L.f_shared > L.f ? L.f_shared : L.f) + 16);
    return union_warps(gu_v, u_stage<true>()) >= 2 && union_warps(dn_v, u_stage<false>()) >= 2;
}

cudaError_t prepare_decode_mma() {
    cudaError_t e = cudaFuncSetAttribute(union_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kUSmemLimit - kUStaticReserve));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(union_mma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kUSmemLimit - kUStaticReserve));
    return e;
}

cudaError_t launch_decode_mma(const LayerDims& L, const moe_weights& W, const uint16_t* x, int T, const Workspace& ws,
                              int num_sms, const Launch& ctx) {
    const int fmax = L.S && L.f_shared > L.f ? L.f_shared : L.f;
    const int vrows = T < kUCols ? T : kUCols;
    UArgs a{};
    a.etab = (const void* const*)ws.etab;
    a.E = L.E;
    a.ulist = ws.ulist;
    a.n_unique = ws.n_unique;
    a.cnt = ws.cnt;
    a.off = ws.off;
    a.perm = ws.perm;
    a.T = T;
    a.k = L.k;
    a.S = L.S;
    a.d = L.d;
    a.f = L.f;
    a.f_sh = L.S ? L.f_shared : L.f;
    a.vrows = vrows;
    a.status = ws.status;
    // gate/up: v = x, out h
    {
        UArgs g = a;
        g.sh_w = (const uint8_t*)W.shared_gate_up;
        g.sh_sc = W.shared_gate_up_scale;
        g.src = x;
        g.src_ld = L.d;
        g.dst = ws.h;
        g.dst_ld = fmax;
        const size_t vb = (size_t)vrows * (2 * (size_t)L.d + 16);
        const int warps = union_warps(vb, u_stage<true>());
        const size_t smem = vb + (size_t)warps * kUStages * u_stage<true>();
        QE_LAUNCH(ctx, MOE_KERNEL_GATEUP,
                  (launch_pdl(L.pdl != 0, union_mma_kernel<true>, dim3(num_sms), dim3(warps * kWarp), smem, ctx.s, g)));
    }
    // down: v = h, out y
    {
        UArgs dn = a;
        dn.sh_w = (const uint8_t*)W.shared_down;
        dn.sh_sc = W.shared_down_scale;
        dn.src = ws.h;
        dn.src_ld = fmax;
        dn.dst = ws.Y;
        dn.dst_ld = L.d;
        const size_t vb = (size_t)vrows * (2 * (size_t)fmax + 16);
        const int warps = union_warps(vb, u_stage<false>());
        const size_t smem = vb + (size_t)warps * kUStages * u_stage<false>();
        QE_LAUNCH(ctx, MOE_KERNEL_DOWN,
                  (launch_pdl(L.pdl != 0, union_mma_kernel<false>, dim3(num_sms), dim3(warps * kWarp), smem, ctx.s, dn)));
    }
    return cudaSuccess;
}

}  // namespace qe
