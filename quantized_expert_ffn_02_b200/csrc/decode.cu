// decode.cu -- K4 (decode expert FFN, int4 and bf16 weights) and K6 (combine).
//
// Batch-union over the bucketed tokens (colibri README, "What's implemented": each unique
// expert is read once and applied to every position routed to it).  Every weight row is
// streamed from HBM once with coalesced 16-byte loads, dequantised in registers and applied to
// the tokens of its bucket; partial dot products are reduced with warp shuffles.
//
// int4 dequantisation.  A 16-byte chunk holds 32 codes (columns 32c .. 32c+31); 32-bit word m
// holds columns 8m .. 8m+7, column 8m+i in bits 4i .. 4i+3.  One LOP3 turns the nibbles at bits
// 0..3 and 16..19 of a word into two 16-bit floats at once (the pair (i, i+4)); shifting the
// word by 4, 8 and 12 brings the other three pairs into place:
//   gate/up  bf16 pair 0x4300 | (nibble ^ 8) = 128 + (s + 8) = 136 + s   (s = the signed code)
//            multiplied by the bf16 activation in a mixed-precision FMA (exact product, fp32
//            sum).  The offset is removed once per row: sum (136 + s) x = sum s x + 136 sum x,
//            with sum x per token computed in fp64 by the router kernel.
//   down     fp16 pair 0x6400 | (nibble ^ 8) = 1032 + s, minus 1032 (one HSUB2) = s exactly,
//            multiplied by the fp16 activation h in a mixed-precision FMA.
// The per-row scale factors out of the dot product and is applied to the reduced sum.
//
// SwiGLU: gate rows 0..f-1, up rows f..2f-1 of the fused matrix (iliria, "What's
// implemented": gate+up fused over one activation; open-1b-verify, "Tensor mapping": w_gate_up
// split at the row boundary).  h = silu(g) * u is stored as fp16 (overflow latches
// MOE_ERR_RANGE).  Down writes y per slot; the combine adds the chosen experts in ascending
// expert index, then the shared expert.
#include "internal.cuh"
#include "decode_common.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace qe {
namespace {

constexpr int kThreads = 256;
constexpr int kGateUpRows = 4;     // gate rows (and the matching up rows) per warp task
constexpr int kDownRows = 8;       // down rows per warp task
constexpr uint32_t kNib = 0x000F000Fu;
constexpr uint32_t kBf16Magic = 0x43084308u;   // bf16 (136 + s) after the nibble flip
constexpr uint32_t kF16Magic = 0x64086408u;    // fp16 (1032 + s) after the nibble flip
constexpr float kBf16Offset = 136.0f;
// int2 codes (four per byte, column 4j + i in bits 2i .. 2i+1): one LOP3 puts (n ^ 2) = s + 2 of
// the codes of columns (i, i+8) of a 32-bit word at bits 0..1 of each 16-bit half:
constexpr uint32_t kCrumb = 0x00030003u;
constexpr uint32_t kBf16Magic2 = 0x43024302u;  // bf16 128 + (s + 2) = 130 + s
constexpr uint32_t kF16Magic2 = 0x64026402u;   // fp16 1024 + (s + 2) = 1026 + s; minus 1026 is s
constexpr float kBf16Offset2 = 130.0f;
// int8 codes (one per byte): bytes 0 and 2 of a word, XOR 0x80, in the low mantissa bits of fp16
// 1024 read 1024 + s + 128 = 1152 + s; minus 1152 is s.
constexpr uint32_t kByte = 0x00FF00FFu;
constexpr uint32_t kF16Magic8 = 0x64806480u;

// Columns per 16-byte chunk of a weight row, and bytes per row of n columns, per weight kind.
template <int WK> struct Kind;
template <> struct Kind<MOE_W_INT4_ROWSCALE> { static constexpr int COLS = 32; __host__ __device__ static size_t bytes(int n) { return (size_t)n / 2; } };
template <> struct Kind<MOE_W_BF16> { static constexpr int COLS = 8; __host__ __device__ static size_t bytes(int n) { return (size_t)n * 2; } };
template <> struct Kind<MOE_W_INT8_ROWSCALE> { static constexpr int COLS = 16; __host__ __device__ static size_t bytes(int n) { return (size_t)n; } };
template <> struct Kind<MOE_W_INT2_ROWSCALE> { static constexpr int COLS = 64; __host__ __device__ static size_t bytes(int n) { return (size_t)n / 4; } };

// bf16 value number i (0..7) of an 8-column x vector
__device__ __forceinline__ unsigned short xhalf(const uint4& v, int i) {
    const uint32_t w = i < 2 ? v.x : i < 4 ? v.y : i < 6 ? v.z : v.w;
    return (unsigned short)((i & 1) ? (w >> 16) : (w & 0xffffu));
}

struct Slots {
    int ntok;      // tokens in the bucket
    int base;      // first routed slot (routed experts) / unused for the shared expert
    bool shared;
};

// Token id and slot of bucket member j.
__device__ __forceinline__ void member(const Slots& b, int j, const int32_t* perm, int k, int T, int& tok,
                                       int& slot) {
    if (b.shared) {
        tok = j;
        slot = T * k + j;
    } else {
        const int p = b.base + j;
        tok = perm[p] / k;
        slot = p;
    }
}

// ---------------------------------------------------------------------------------------
// gate/up + SiLU
// ---------------------------------------------------------------------------------------
template <int WK, int TG>
__global__ void __launch_bounds__(kThreads, 2)
gateup_kernel(const uint8_t* __restrict__ gate_up, const float* __restrict__ gu_scale,
              const uint8_t* __restrict__ sh_gate_up, const float* __restrict__ sh_gu_scale,
              const uint16_t* __restrict__ x, const double* __restrict__ xsum, int T, int k, int d, int f,
              int f_sh, int S, const int32_t* __restrict__ ulist, const int32_t* __restrict__ n_unique_p,
              const int32_t* __restrict__ cnt, const int32_t* __restrict__ off, const int32_t* __restrict__ perm,
              uint16_t* __restrict__ h, int fmax, int* status, const void* const* __restrict__ etab, int E) {
    // Launched with programmatic dependent launch after the previous kernel of the layer: wait
    // for its results before reading anything, then let the next kernel launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int R = kGateUpRows;
    constexpr int COLS = Kind<WK>::COLS;                          // columns per 16-byte chunk
    constexpr int XV = COLS / 8;                                  // 16-byte x vectors per chunk
    const int lane = threadIdx.x % kWarp;
    const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
    const int nwarps = gridDim.x * blockDim.x / kWarp;
    const int n_unique = *n_unique_p;
    const int per_routed = f / R;
    const int n_tasks = n_unique * per_routed + (S ? f_sh / R : 0);
    const int nchunk = d / COLS;
    const size_t rowbytes = Kind<WK>::bytes(d);

    for (int task = gwarp; task < n_tasks; task += nwarps) {
        const uint8_t* W;
        const float* sc;
        int fe, r0;
        Slots b;
        if (task < n_unique * per_routed) {
            const int e = ulist[task / per_routed];
            r0 = (task % per_routed) * R;
            fe = f;
            W = ex_gate_up(etab, E, e);
            sc = WK != MOE_W_BF16 ? ex_gu_scale(etab, E, e) : nullptr;
            b = Slots{cnt[e], off[e], false};
        } else {
            r0 = (task - n_unique * per_routed) * R;
            fe = f_sh;
            W = sh_gate_up;
            sc = sh_gu_scale;
            b = Slots{T, 0, true};
        }
        for (int g0 = 0; g0 < b.ntok; g0 += TG) {
            const int ng = min(TG, b.ntok - g0);
            int tok[TG], slot[TG];
#pragma unroll
            for (int j = 0; j < TG; ++j) {
                tok[j] = 0;
                slot[j] = 0;
                if (j < ng) member(b, g0 + j, perm, k, T, tok[j], slot[j]);
            }
            float acc[2 * R][TG];
#pragma unroll
            for (int rr = 0; rr < 2 * R; ++rr)
#pragma unroll
                for (int j = 0; j < TG; ++j) acc[rr][j] = 0.0f;

            // the next chunk's rows are in flight while this chunk is multiplied
            uint4 wn[2 * R];
            auto load_rows = [&](int c, uint4 (&dst)[2 * R]) {
#pragma unroll
                for (int rr = 0; rr < 2 * R; ++rr) {
                    const int row = rr < R ? r0 + rr : fe + r0 + (rr - R);
                    dst[rr] = ld_stream16(W + (size_t)row * rowbytes + (size_t)c * 16);
                }
            };
            // (one-token passes only: with more tokens per pass the registers run out)
            constexpr bool kAhead = TG == 1;
            if (kAhead && lane < nchunk) load_rows(lane, wn);
            for (int c = lane; c < nchunk; c += kWarp) {
                uint4 wv[2 * R];
                if (kAhead) {
#pragma unroll
                    for (int rr = 0; rr < 2 * R; ++rr) wv[rr] = wn[rr];
                    if (c + kWarp < nchunk) load_rows(c + kWarp, wn);
                } else {
                    load_rows(c, wv);
                }
#pragma unroll
                for (int j = 0; j < TG; ++j) {
                    if (j < ng) {
                        uint4 xv[XV];
#pragma unroll
                        for (int m = 0; m < XV; ++m)
                            xv[m] = ld_ro16(x + (size_t)tok[j] * d + (size_t)c * COLS + 8 * m);
#pragma unroll
                        for (int rr = 0; rr < 2 * R; ++rr) {
                            float a = acc[rr][j];
                            if (WK == MOE_W_INT4_ROWSCALE) {
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    const uint32_t w = words[m];
                                    unsigned short a0, a1, a2, a3, a4, a5, a6, a7;
                                    halves(lop_sel_xor(w, kNib, kBf16Magic), a0, a4);
                                    halves(lop_sel_xor(w >> 4, kNib, kBf16Magic), a1, a5);
                                    halves(lop_sel_xor(w >> 8, kNib, kBf16Magic), a2, a6);
                                    halves(lop_sel_xor(w >> 12, kNib, kBf16Magic), a3, a7);
                                    unsigned short x0, x1, x2, x3, x4, x5, x6, x7;
                                    halves(xv[m].x, x0, x1);
                                    halves(xv[m].y, x2, x3);
                                    halves(xv[m].z, x4, x5);
                                    halves(xv[m].w, x6, x7);
                                    a = fma_bf16(a0, x0, a);
                                    a = fma_bf16(a1, x1, a);
                                    a = fma_bf16(a2, x2, a);
                                    a = fma_bf16(a3, x3, a);
                                    a = fma_bf16(a4, x4, a);
                                    a = fma_bf16(a5, x5, a);
                                    a = fma_bf16(a6, x6, a);
                                    a = fma_bf16(a7, x7, a);
                                }
                            } else if (WK == MOE_W_INT2_ROWSCALE) {
                                // word m: columns 16m .. 16m+15 (x vectors 2m and 2m+1)
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
#pragma unroll
                                    for (int i = 0; i < 8; ++i) {
                                        unsigned short lo, hi;
                                        halves(lop_sel_xor(words[m] >> (2 * i), kCrumb, kBf16Magic2), lo, hi);
                                        a = fma_bf16(lo, xhalf(xv[2 * m], i), a);
                                        a = fma_bf16(hi, xhalf(xv[2 * m + 1], i), a);
                                    }
                                }
                            } else if (WK == MOE_W_INT8_ROWSCALE) {
                                // word m: columns 4m .. 4m+3; the codes convert exactly to fp32
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        const float q = (float)((int)(words[m] << (24 - 8 * i)) >> 24);
                                        a = fmaf(q, bf16_bits_to_f32(xhalf(xv[m >> 1], 4 * (m & 1) + i)), a);
                                    }
                                }
                            } else {
                                const uint32_t ws[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
                                const uint32_t xs[4] = {xv[0].x, xv[0].y, xv[0].z, xv[0].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    unsigned short wl, wh, xl, xh;
                                    halves(ws[m], wl, wh);
                                    halves(xs[m], xl, xh);
                                    a = fma_bf16(wl, xl, a);
                                    a = fma_bf16(wh, xh, a);
                                }
                            }
                            acc[rr][j] = a;
                        }
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < 2 * R; ++rr)
#pragma unroll
                for (int j = 0; j < TG; ++j) acc[rr][j] = warp_sum(acc[rr][j]);
            // lanes 0..R-1 finish one row each
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                if (lane == rr) {
                    const int r = r0 + rr;
#pragma unroll
                    for (int j = 0; j < TG; ++j) {
                        if (j < ng) {
                            float g = acc[rr][j], u = acc[R + rr][j];
                            if (WK != MOE_W_BF16) {
                                const float off = WK == MOE_W_INT4_ROWSCALE ? kBf16Offset * (float)xsum[tok[j]]
                                                  : WK == MOE_W_INT2_ROWSCALE ? kBf16Offset2 * (float)xsum[tok[j]]
                                                                              : 0.0f;
                                g = sc[r] * (g - off);
                                u = sc[fe + r] * (u - off);
                            }
                            const float hv = g / (1.0f + expf(-g)) * u;
                            const __half hh = __float2half_rn(hv);
                            if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(status, MOE_ERR_RANGE);
                            h[(size_t)slot[j] * fmax + r] = __half_as_ushort(hh);
                        }
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// down: Y[slot][j] = scale[j] * sum_r q[j][r] h[slot][r]
// ---------------------------------------------------------------------------------------
template <int WK, int TG>
__global__ void __launch_bounds__(kThreads, 2)
down_kernel(const uint8_t* __restrict__ down, const float* __restrict__ dn_scale,
            const uint8_t* __restrict__ sh_down, const float* __restrict__ sh_dn_scale,
            const uint16_t* __restrict__ h, int fmax, int T, int k, int d, int f, int f_sh, int S,
            const int32_t* __restrict__ ulist, const int32_t* __restrict__ n_unique_p,
            const int32_t* __restrict__ cnt, const int32_t* __restrict__ off, const int32_t* __restrict__ perm,
            float* __restrict__ Y, const void* const* __restrict__ etab, int E) {
    // Launched with programmatic dependent launch after the previous kernel of the layer: wait
    // for its results before reading anything, then let the next kernel launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int R = kDownRows;
    constexpr int COLS = Kind<WK>::COLS;
    constexpr int HV = COLS / 8;      // 16-byte h vectors per chunk
    const int lane = threadIdx.x % kWarp;
    const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
    const int nwarps = gridDim.x * blockDim.x / kWarp;
    const int n_unique = *n_unique_p;
    const int per = d / R;
    const int n_tasks = (n_unique + (S ? 1 : 0)) * per;

    for (int task = gwarp; task < n_tasks; task += nwarps) {
        const int u = task / per;
        const int j0 = (task % per) * R;
        const uint8_t* W;
        const float* sc;
        int fe;
        Slots b;
        if (u < n_unique) {
            const int e = ulist[u];
            fe = f;
            W = ex_down(etab, E, e);
            sc = WK != MOE_W_BF16 ? ex_dn_scale(etab, E, e) : nullptr;
            b = Slots{cnt[e], off[e], false};
        } else {
            fe = f_sh;
            W = sh_down;
            sc = sh_dn_scale;
            b = Slots{T, 0, true};
        }
        const size_t rowbytes = Kind<WK>::bytes(fe);
        const int nchunk = fe / COLS;
        for (int g0 = 0; g0 < b.ntok; g0 += TG) {
            const int ng = min(TG, b.ntok - g0);
            int slot[TG];
#pragma unroll
            for (int j = 0; j < TG; ++j) {
                int tk = 0;
                slot[j] = 0;
                if (j < ng) member(b, g0 + j, perm, k, T, tk, slot[j]);
            }
            float acc[R][TG];
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
#pragma unroll
                for (int j = 0; j < TG; ++j) acc[rr][j] = 0.0f;
            // the next chunk's rows are in flight while this chunk is multiplied
            // (one-token passes only: with more tokens per pass the registers run out)
            constexpr bool kAhead = TG == 1;
            uint4 wn[R];
            if (kAhead && lane < nchunk)
#pragma unroll
                for (int rr = 0; rr < R; ++rr) wn[rr] = ld_stream16(W + (size_t)(j0 + rr) * rowbytes + (size_t)lane * 16);
            for (int c = lane; c < nchunk; c += kWarp) {
                uint4 wv[R];
                if (kAhead) {
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) wv[rr] = wn[rr];
                    if (c + kWarp < nchunk)
#pragma unroll
                        for (int rr = 0; rr < R; ++rr)
                            wn[rr] = ld_stream16(W + (size_t)(j0 + rr) * rowbytes + (size_t)(c + kWarp) * 16);
                } else {
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) wv[rr] = ld_stream16(W + (size_t)(j0 + rr) * rowbytes + (size_t)c * 16);
                }
#pragma unroll
                for (int j = 0; j < TG; ++j) {
                    if (j < ng) {
                        uint4 hv[HV];
#pragma unroll
                        for (int m = 0; m < HV; ++m) hv[m] = ld_ro16(h + (size_t)slot[j] * fmax + (size_t)c * COLS + 8 * m);
#pragma unroll
                        for (int rr = 0; rr < R; ++rr) {
                            float a = acc[rr][j];
                            if (WK == MOE_W_INT4_ROWSCALE) {
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    const uint32_t w = words[m];
                                    unsigned short s0, s1, s2, s3, s4, s5, s6, s7;
                                    halves(hsub2_u32(lop_sel_xor(w, kNib, kF16Magic), kF16Magic), s0, s4);
                                    halves(hsub2_u32(lop_sel_xor(w >> 4, kNib, kF16Magic), kF16Magic), s1, s5);
                                    halves(hsub2_u32(lop_sel_xor(w >> 8, kNib, kF16Magic), kF16Magic), s2, s6);
                                    halves(hsub2_u32(lop_sel_xor(w >> 12, kNib, kF16Magic), kF16Magic), s3, s7);
                                    unsigned short h0, h1, h2, h3, h4, h5, h6, h7;
                                    halves(hv[m].x, h0, h1);
                                    halves(hv[m].y, h2, h3);
                                    halves(hv[m].z, h4, h5);
                                    halves(hv[m].w, h6, h7);
                                    a = fma_f16(s0, h0, a);
                                    a = fma_f16(s1, h1, a);
                                    a = fma_f16(s2, h2, a);
                                    a = fma_f16(s3, h3, a);
                                    a = fma_f16(s4, h4, a);
                                    a = fma_f16(s5, h5, a);
                                    a = fma_f16(s6, h6, a);
                                    a = fma_f16(s7, h7, a);
                                }
                            } else if (WK == MOE_W_INT2_ROWSCALE) {
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
#pragma unroll
                                    for (int i = 0; i < 8; ++i) {
                                        unsigned short lo, hi;
                                        halves(hsub2_u32(lop_sel_xor(words[m] >> (2 * i), kCrumb, kF16Magic2), kF16Magic2),
                                               lo, hi);
                                        a = fma_f16(lo, xhalf(hv[2 * m], i), a);
                                        a = fma_f16(hi, xhalf(hv[2 * m + 1], i), a);
                                    }
                                }
                            } else if (WK == MOE_W_INT8_ROWSCALE) {
                                const uint32_t words[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    unsigned short s0, s1, s2, s3;
                                    halves(hsub2_u32(lop_sel_xor(words[m], kByte, kF16Magic8), kF16Magic8), s0, s2);
                                    halves(hsub2_u32(lop_sel_xor(words[m] >> 8, kByte, kF16Magic8), kF16Magic8), s1, s3);
                                    const int b = 4 * (m & 1);
                                    a = fma_f16(s0, xhalf(hv[m >> 1], b), a);
                                    a = fma_f16(s1, xhalf(hv[m >> 1], b + 1), a);
                                    a = fma_f16(s2, xhalf(hv[m >> 1], b + 2), a);
                                    a = fma_f16(s3, xhalf(hv[m >> 1], b + 3), a);
                                }
                            } else {
                                const uint32_t ws[4] = {wv[rr].x, wv[rr].y, wv[rr].z, wv[rr].w};
                                const uint32_t hs[4] = {hv[0].x, hv[0].y, hv[0].z, hv[0].w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hs[m]));
                                    a = fmaf(__uint_as_float(ws[m] << 16), hf.x, a);
                                    a = fmaf(__uint_as_float(ws[m] & 0xffff0000u), hf.y, a);
                                }
                            }
                            acc[rr][j] = a;
                        }
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
#pragma unroll
                for (int j = 0; j < TG; ++j) acc[rr][j] = warp_sum(acc[rr][j]);
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                if (lane == rr) {
                    const int jr = j0 + rr;
                    const float s = WK != MOE_W_BF16 ? sc[jr] : 1.0f;
#pragma unroll
                    for (int j = 0; j < TG; ++j)
                        if (j < ng) Y[(size_t)slot[j] * d + jr] = s * acc[rr][j];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// combine: out[t] = sum over the chosen experts in ascending index of w * Y + shared
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float* __restrict__ Y, const float* __restrict__ wts, const int32_t* __restrict__ asc,
               const int32_t* __restrict__ slot_of, int T, int k, int d, int S, void* __restrict__ out,
               int out_bf16) {
    // Launched with programmatic dependent launch after the previous kernel of the layer: wait
    // for its results before reading anything, then let the next kernel launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int t = blockIdx.y;
    const int j4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (j4 * 4 >= d) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < k; ++p) {
        const int r = asc[(size_t)t * k + p];
        const float w = wts[(size_t)t * k + r];
        const int slot = slot_of[(size_t)t * k + r];
        if (slot < 0) continue;                   // dropped by adaptive top-p
        const float4 y = reinterpret_cast<const float4*>(Y + (size_t)slot * d)[j4];
        acc.x = fmaf(w, y.x, acc.x);
        acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z);
        acc.w = fmaf(w, y.w, acc.w);
    }
    if (S) {
        const float4 y = reinterpret_cast<const float4*>(Y + (size_t)(T * k + t) * d)[j4];
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
    }
    if (out_bf16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t*>(&lo);
        v.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + (size_t)t * d)[j4] = v;
    } else {
        reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)t * d)[j4] = acc;
    }
}

template <int WK, int TG>
cudaError_t launch_experts_t(const LayerDims& L, const moe_weights& W, const uint16_t* x, int T,
                             const Workspace& ws, int num_sms, const Launch& ctx) {
    const int fmax = L.S && L.f_shared > L.f ? L.f_shared : L.f;
    const unsigned grid = (unsigned)num_sms * 2;
    const bool pdl = L.pdl != 0;
    QE_LAUNCH(ctx, MOE_KERNEL_GATEUP,
              (dec::launch_pdl(pdl, gateup_kernel<WK, TG>, dim3(grid), dim3(kThreads), 0, ctx.s,
                  (const uint8_t*)W.gate_up, W.gate_up_scale, (const uint8_t*)W.shared_gate_up, W.shared_gate_up_scale,
                  x, (const double*)ws.xsum, T, L.k, L.d, L.f, L.f_shared, L.S, (const int32_t*)ws.ulist,
                  (const int32_t*)ws.n_unique, (const int32_t*)ws.cnt, (const int32_t*)ws.off, (const int32_t*)ws.perm,
                  ws.h, fmax, ws.status, (const void* const*)ws.etab, L.E)));
    QE_LAUNCH(ctx, MOE_KERNEL_DOWN,
              (dec::launch_pdl(pdl, down_kernel<WK, TG>, dim3(grid), dim3(kThreads), 0, ctx.s,
                  (const uint8_t*)W.down, W.down_scale, (const uint8_t*)W.shared_down, W.shared_down_scale,
                  (const uint16_t*)ws.h, fmax, T, L.k, L.d, L.f, L.f_shared, L.S, (const int32_t*)ws.ulist,
                  (const int32_t*)ws.n_unique, (const int32_t*)ws.cnt, (const int32_t*)ws.off, (const int32_t*)ws.perm,
                  ws.Y, (const void* const*)ws.etab, L.E)));
    return cudaSuccess;
}

}  // namespace


cudaError_t launch_decode_experts(const LayerDims& L, const moe_weights& W, const uint16_t* x, int T,
                                  const Workspace& ws, int num_sms, const Launch& ctx) {
    if (T == 0) return cudaSuccess;
    // Tokens per pass over a row.  Small batches: one, with the next chunk's rows in flight.
    // Larger batches: two, which keeps the passes of the shared expert (every token) few; either
    // way the register count allows two CTAs per SM, and a bucket larger than the group takes
    // more passes over rows that are by then in L2.
    if (L.wkind == MOE_W_INT4_ROWSCALE)
        return T <= 4 ? launch_experts_t<MOE_W_INT4_ROWSCALE, 1>(L, W, x, T, ws, num_sms, ctx)
                      : launch_experts_t<MOE_W_INT4_ROWSCALE, 2>(L, W, x, T, ws, num_sms, ctx);
    if (L.wkind == MOE_W_INT8_ROWSCALE)
        return T <= 4 ? launch_experts_t<MOE_W_INT8_ROWSCALE, 1>(L, W, x, T, ws, num_sms, ctx)
                      : launch_experts_t<MOE_W_INT8_ROWSCALE, 2>(L, W, x, T, ws, num_sms, ctx);
    if (L.wkind == MOE_W_INT2_ROWSCALE)
        return T <= 4 ? launch_experts_t<MOE_W_INT2_ROWSCALE, 1>(L, W, x, T, ws, num_sms, ctx)
                      : launch_experts_t<MOE_W_INT2_ROWSCALE, 2>(L, W, x, T, ws, num_sms, ctx);
    return T <= 4 ? launch_experts_t<MOE_W_BF16, 1>(L, W, x, T, ws, num_sms, ctx)
                  : launch_experts_t<MOE_W_BF16, 2>(L, W, x, T, ws, num_sms, ctx);
}

cudaError_t launch_combine(const LayerDims& L, int T, const Workspace& ws, void* out, const Launch& ctx) {
    if (T == 0) return cudaSuccess;
    dim3 grid((unsigned)((L.d / 4 + kThreads - 1) / kThreads), (unsigned)T);
    QE_LAUNCH(ctx, MOE_KERNEL_COMBINE,
              (dec::launch_pdl(L.pdl != 0, combine_kernel, grid, dim3(kThreads), 0, ctx.s, (const float*)ws.Y,
                               (const float*)ws.wts, (const int32_t*)ws.asc, (const int32_t*)ws.slot_of, T, L.k, L.d,
                               L.S, out, L.out_bf16)));
    return cudaSuccess;
}

}  // namespace qe
