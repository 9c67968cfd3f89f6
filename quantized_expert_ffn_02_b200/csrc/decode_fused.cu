// decode_fused.cu -- the whole layer for one token with int4 experts, in one cooperative launch.
//
// For one token the layer reads each weight byte once, so its time is the time to stream the
// router matrix and k + 1 experts from HBM.  Separate kernels for the router, gate/up and down
// each pay the ramp of a fresh grid and leave HBM idle while the previous grid drains; here one
// persistent CTA per SM runs the steps back to back and keeps its copies in flight
// across the joins.  Each warp streams its weight rows through a private two-stage ring of TMA
// bulk copies (a gate row, the matching up row and two 16-byte slivers holding their scales per
// stage).  Up to 16 warps per CTA: as many as the rings fit in shared memory beside x.
//
// Shared memory: x as the MMA operand (x~ below), one block per lane holding the lane's groups in
// the order it visits them, then the rings.  Phase A parks the plain bf16 x in the rings' last
// stage; phase B keeps the router pieces, keys and logits at the start of the idle rings.
//
//   A  router + shared expert.  One bulk copy brings x in while each warp's first router piece
//      (one expert x 1024 columns, coalesced loads) is in flight.  The CTA builds x~ from x, the
//      warps compute their router pieces in fp64 and store them, the CTA arrives on grid
//      barrier 0, and the warps reduce the shared expert's row pairs (they need no routing) while
//      the other CTAs arrive.
//   B  selection, by the whole CTA: one bulk copy gathers every piece; thread e sums expert e's
//      pieces (the same order in every CTA, so every CTA selects the same experts) and forms an
//      order-preserving integer key; the k best of each warp's 32 experts become candidates, and
//      each candidate's rank among the candidates is its overall rank.  The k experts (ascending)
//      and their gate weights go to shared memory,  (the gate/up stream is
//      marked evict-first, so the shared expert's down rows pulled into L2 in A stay there).
//   C  routed gate/up: row pairs of the k experts, strided over every warp of the grid;
//      h = SiLU(gate) * up in fp16 (global, L2), the SiLU of 32 row pairs at a time.  A warp that
//      has finished its row pairs queues its first down rows (they do not depend on h), then the
//      CTA arrives on grid barrier 1, after which every h is complete.
//   D  down + combine: CTA b owns output rows [b d / G, (b + 1) d / G) of every slot (the k
//      routed experts in ascending index order, then the shared expert); its warps split the
//      (slot, row) list, and the CTA adds the slots with their gate weights and stores y.
//
// The dot products run on the tensor cores (mma.sync m16n8k16, fp16 operands, fp32
// accumulation) -- not to reach tensor-core throughput, which a matrix-vector product cannot use,
// but because the same sums on the FP32 pipe cost about two instructions per weight and lane and
// bound the kernel by instruction issue instead of HBM.  One MMA takes the 16 rows
// {8 K-segments of the gate row, the same 8 segments of the up row} against B = the 8 matching
// segments of x, one per column; the diagonal of the 8 x 8 product blocks is the two dot products
// (the off-diagonal terms are discarded).  Lane (g, c) of the warp feeds segment g, so it only
// ever touches x and weights of its own segment, at the K positions of its own quarter.
//
// Dequantisation: a code s = n - 16 [n >= 8] is stored as the nibble n; n ^ 8 = s + 8.  One LOP3
// builds the pair (n_i ^ 8, n_{i+4} ^ 8) at fp16 mantissa bits 0..3 with a zero exponent -- the
// exact fp16 value (s + 8) 2^-24 -- or at bits 4..7, the exact value (s + 8) 2^-20; one shift by
// 8 bits reaches the other two nibble pairs, so 8 codes cost one shift and four LOP3s.  The x
// entries that meet the 2^-20 codes are stored scaled by 2^-4, so every product is
// (s + 8) x 2^-24, exact, and the fp32 sums give sum s x = 2^24 D - 8 sum x.  x enters as fp16
// x 2^sigma, with sigma a per-token power of two that puts max|x| in [2^14, 2^15): every bf16
// value in that range converts exactly.  h (fp16 already) is scaled the same way per slot.  The
// router logits accumulate in fp64 on the FP64 pipe.
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
constexpr int kFzMaxThreads = kFzMaxWarps * kWarp;
constexpr int kFzStages = 2;
constexpr int kFzMaxSlots = 10;       // k routed experts + the shared one
constexpr int kFzMaxPer = 8;          // experts per lane in the selection: E <= 256
constexpr int kFzRowsMax = 64;        // output rows per CTA (one token; 48 for two)
constexpr int kFzDnRowsMax = 8;       // down rows per stage
constexpr int kFzScRegs = 3;          // down-row scales per lane: up to 96 (slot, row) items per warp
constexpr size_t kSmemLimit = 227 * 1024;
// output rows per CTA and the kernel's static shared memory (rounded up), for nt tokens
constexpr int fz_rows_max(int nt) { return nt == 1 ? kFzRowsMax : 48; }
constexpr size_t fz_static_reserve(int nt) { return nt == 1 ? 6144 : 8192; }
// the element i of a per-token register array, without a local-memory copy for a runtime index
template <int N, typename V>
__device__ __forceinline__ V pick_tok(const V (&v)[N], int i) {
    V r = v[0];
#pragma unroll
    for (int j = 1; j < N; ++j)
        if (i == j) r = v[j];
    return r;
}

struct FusedArgs {
    const float* router_w;            // [E][d] fp32
    const float* bias;                // [E] selection bias (sigmoid router) or null
    const uint16_t* x;                // [d] bf16
    const uint8_t* sh_gate_up;        // [2f][d/2]
    const float* sh_gu_scale;         // [2f]
    const uint8_t* sh_down;           // [d][f/2]
    const float* sh_dn_scale;         // [d]
    const void* const* etab;          // [4][E] the routed experts' gate/up, its scales, down, its scales
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
    unsigned long long* trace;        // [CTA][16] %globaltimer at the phase boundaries (or null)
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
// Returns the count before the arrival.  One thread calls it.  (A fire-and-forget add in its
// place measured slower: the other CTAs saw the last arrival about 1 us later.)
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
// L2 cache policies: streamed weight rows are read once (evict first); the down rows prefetched
// for phase D should outlive them (normal priority).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Bulk copy global -> shared with an L2 cache policy, completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
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

// ---------------------------------------------------------------------------------------
// The tensor-core dot products
// ---------------------------------------------------------------------------------------
// D += A B for one m16n8k16 tile, fp16 operands, fp32 accumulators.  Fragments (lane = 4 g + c):
// a0 = A[g][2c, 2c+1], a1 = A[g+8][2c, 2c+1], a2 = A[g][2c+8, 2c+9], a3 = A[g+8][2c+8, 2c+9];
// b0 = B[2c, 2c+1][g], b1 = B[2c+8, 2c+9][g]; d = D[g][2c, 2c+1], D[g+8][2c, 2c+1].
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Codes of columns (i, i+4) of a 32-bit word (nibble i = column i) as the fp16 pair
// ((s_i + 8) 2^-24, (s_{i+4} + 8) 2^-24) for i = 0 (nib_lo) or (s + 8) 2^-20 for i = 1 (nib_hi);
// of w >> 8, the same for i = 2 and 3.
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) { return lop_sel_xor(w, 0x000F000Fu, 0x00080008u); }
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) { return lop_sel_xor(w, 0x00F000F0u, 0x00800080u); }

// The 16-byte group a lane reads at step j of a row: its groups are visited from a lane-dependent
// start so that the 8 lanes of each shared-memory phase hit 8 different bank quads (checked for
// every width the kernel takes).
template <int NDK>
__device__ __forceinline__ int gu_rot(int lane) {
    const int g = lane >> 2, c = lane & 3;
    if (NDK % 2) return 0;
    if (NDK == 4) return (c >> 1) + 2 * (g & 1);
    if (NDK == 8) return (g & 1) + 2 * c;
    return g & 1;
}
template <int NF>
__device__ __forceinline__ int dn_rot(int lane) {
    return gu_rot<NF>(lane);      // a down row's lane quarter has the same geometry
}

// 8 bf16 (or fp16) values of one 8-column group, as the four operand pairs of that group:
// (col 0, col 4), (col 1, col 5) x 2^-4, (col 2, col 6), (col 3, col 7) x 2^-4, each scaled by
// 2^e (fp32 arithmetic, then one rounding to fp16; exact for values in fp16's normal range).
__device__ __forceinline__ void pairs_from_bf16(uint4 v, float s, float s16, uint32_t* p, float& sum) {
    const float c0 = __uint_as_float(v.x << 16), c1 = __uint_as_float(v.x & 0xffff0000u);
    const float c2 = __uint_as_float(v.y << 16), c3 = __uint_as_float(v.y & 0xffff0000u);
    const float c4 = __uint_as_float(v.z << 16), c5 = __uint_as_float(v.z & 0xffff0000u);
    const float c6 = __uint_as_float(v.w << 16), c7 = __uint_as_float(v.w & 0xffff0000u);
    const __half2 p0 = __floats2half2_rn(c0 * s, c4 * s), p1 = __floats2half2_rn(c1 * s16, c5 * s16);
    const __half2 p2 = __floats2half2_rn(c2 * s, c6 * s), p3 = __floats2half2_rn(c3 * s16, c7 * s16);
    p[0] = *reinterpret_cast<const uint32_t*>(&p0);
    p[1] = *reinterpret_cast<const uint32_t*>(&p1);
    p[2] = *reinterpret_cast<const uint32_t*>(&p2);
    p[3] = *reinterpret_cast<const uint32_t*>(&p3);
    // the sum of the scaled values the MMA sees at the unscaled positions (fp16-rounded)
    const float2 f0 = __half22float2(p0), f2 = __half22float2(p2);
    const float2 f1 = __half22float2(p1), f3 = __half22float2(p3);
    sum += (f0.x + f0.y) + (f2.x + f2.y) + 16.0f * ((f1.x + f1.y) + (f3.x + f3.y));
}
__device__ __forceinline__ void pairs_from_f16(uint4 v, float s, float s16, uint32_t* p, float& sum) {
    const uint32_t q[4] = {__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                           __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&q[i]));
        const float m = (i & 1) ? s16 : s;
        const __half2 r = __floats2half2_rn(f.x * m, f.y * m);
        p[i] = *reinterpret_cast<const uint32_t*>(&r);
        const float2 b = __half22float2(r);
        sum += (i & 1) ? 16.0f * (b.x + b.y) : (b.x + b.y);
    }
}
// 2^e as a float for |e| <= 126.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }
// The power of two that moves max|v| (v > 0, finite) into [2^14, 2^15), clamped to [-100, 100];
// 0 for v == 0.
__device__ __forceinline__ int scale_exp(float vmax) {
    if (!(vmax > 0.0f) || !isfinite(vmax)) return 0;
    const int e = (int)((__float_as_uint(vmax) >> 23) & 0xff) - 127;   // floor(log2 vmax), vmax normal in fp32
    return max(-100, min(100, 14 - e));
}

// Where h[r] of a slot is kept: the lane that reads r in phase D owns the 8-value chunks
// [L cpl, (L + 1) cpl) of the row (cpl = f / 256 chunks per lane), and chunk m of every lane is
// stored at m * 32 + L, so that each 16-byte load of the warp reads 512 contiguous bytes.
template <int F>
__device__ __forceinline__ int h_pos(int r) {
    constexpr int cpl = F / 256;
    const int L = r / (8 * cpl), m = (r >> 3) % cpl;
    return (m * kWarp + L) * 8 + (r & 7);
}

// Independent accumulator chains per dot product: an MMA's result feeds the next MMA of its chain
// only, so a chain's latency is paid every kChains MMAs.
constexpr int kChains = 4;

// The weight kinds of this kernel.  A "group" is the 16 bytes of a weight row that a lane loads at
// once: 32 int4 codes (8 K steps of the MMA for a row pair) or 8 bf16 values (2 K steps).  XR is the
// number of 32-bit operand registers of x (or h) that one group meets.
template <int WK> struct FzKind;
template <> struct FzKind<MOE_W_INT4_ROWSCALE> {
    static constexpr int COLS = 32, XR = 16, HR = 16;
    static constexpr int row_bytes(int cols) { return cols / 2; }
};
template <> struct FzKind<MOE_W_BF16> {
    static constexpr int COLS = 8, XR = 4, HR = 8;     // h: 4 registers of bf16 high parts, 4 of low parts
    static constexpr int row_bytes(int cols) { return cols * 2; }
};

// Diagonal of the two 8 x 8 blocks held by the warp's D fragments (the chains added up): this
// lane's part of (rows 0..7 . columns) and (rows 8..15 . columns); 0 for lanes that hold no
// diagonal entry.
__device__ __forceinline__ float2 diag_part(const float (&acc)[kChains][4], int lane) {
    const int g = lane >> 2, c = lane & 3;
    if (c != (g >> 1)) return make_float2(0.0f, 0.0f);
    float e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float t = 0.0f;
#pragma unroll
        for (int ch = 0; ch < kChains; ++ch) t += acc[ch][i];
        e[i] = t;
    }
    return (g & 1) ? make_float2(e[1], e[3]) : make_float2(e[0], e[2]);
}

// The same tile with bf16 operands (the bf16 weight kind).
__device__ __forceinline__ void mma16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two rows (A rows 0..7: the first row's 8 K-segments, rows 8..15: the second row's) times the
// lane's operand registers xr: this lane's part of both dot products (see diag_part).  G groups
// per lane, visited from the lane's rotation; lane_off is the byte offset of its segment quarter.
//   int4: 2^24 times the sums of (s + 8) x~ (codes decoded in place, see nib_lo / nib_hi);
//   bf16: the sums of w x (the weights are the MMA operand as they are).
// For the down rows the operand holds h~ (int4) or h split into bf16 high and low parts (bf16,
// two MMAs per K step).
template <int WK, int G, int XR, bool SPLIT>
__device__ __forceinline__ float2 rows_mma(uint32_t rowA, uint32_t rowB, uint32_t lane_off, int rot,
                                           const uint32_t (&xr)[G][XR], int lane) {
    float acc[kChains][4] = {};
    int chain = 0;
#pragma unroll
    for (int j = 0; j < G; ++j) {
        int q = j + rot;
        if (q >= G) q -= G;
        const uint32_t off = lane_off + 16u * (uint32_t)q;
        const uint4 A = lds16(rowA + off), B = lds16(rowB + off);
        const uint32_t aw[4] = {A.x, A.y, A.z, A.w}, bw[4] = {B.x, B.y, B.z, B.w};
        if (WK == MOE_W_INT4_ROWSCALE) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                mma16816(acc[chain++ % kChains], nib_lo(aw[w]), nib_lo(bw[w]), nib_hi(aw[w]), nib_hi(bw[w]),
                         xr[j][4 * w], xr[j][4 * w + 1]);
                const uint32_t a8 = aw[w] >> 8, b8 = bw[w] >> 8;
                mma16816(acc[chain++ % kChains], nib_lo(a8), nib_lo(b8), nib_hi(a8), nib_hi(b8), xr[j][4 * w + 2],
                         xr[j][4 * w + 3]);
            }
        } else {
            // K step s: columns 4s .. 4s+3 of the group; k-slots (2c, 2c+1) take the first pair
#pragma unroll
            for (int st = 0; st < 2; ++st) {
                mma16816_bf16(acc[chain++ % kChains], aw[2 * st], bw[2 * st], aw[2 * st + 1], bw[2 * st + 1],
                              xr[j][2 * st], xr[j][2 * st + 1]);
                if (SPLIT)
                    mma16816_bf16(acc[chain++ % kChains], aw[2 * st], bw[2 * st], aw[2 * st + 1], bw[2 * st + 1],
                                  xr[j][4 + 2 * st], xr[j][4 + 2 * st + 1]);
            }
        }
    }
    return diag_part(acc, lane);
}

// The same two-row product with the operand of x read from this lane's block in shared memory
// (xblk), one 16-byte group at a time: the loop over the groups stays rolled, so the code stays
// small and the operand takes no long-lived registers.
template <int WK, int G>
__device__ __forceinline__ float2 rows_mma_x(uint32_t rowA, uint32_t rowB, uint32_t lane_off, int rot, uint32_t xblk,
                                             int lane) {
    float acc[kChains][4] = {};
    int q = rot;
#pragma unroll 1
    for (int j = 0; j < G; ++j) {
        const uint32_t off = lane_off + 16u * (uint32_t)q;
        if (++q == G) q = 0;
        const uint4 A = lds16(rowA + off), B = lds16(rowB + off);
        const uint32_t aw[4] = {A.x, A.y, A.z, A.w}, bw[4] = {B.x, B.y, B.z, B.w};
        if (WK == MOE_W_INT4_ROWSCALE) {
            uint32_t xv[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint4 v = lds16(xblk + (uint32_t)(64 * j + 16 * m));
                xv[4 * m] = v.x;
                xv[4 * m + 1] = v.y;
                xv[4 * m + 2] = v.z;
                xv[4 * m + 3] = v.w;
            }
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                mma16816(acc[w], nib_lo(aw[w]), nib_lo(bw[w]), nib_hi(aw[w]), nib_hi(bw[w]), xv[4 * w], xv[4 * w + 1]);
                const uint32_t a8 = aw[w] >> 8, b8 = bw[w] >> 8;
                mma16816(acc[w], nib_lo(a8), nib_lo(b8), nib_hi(a8), nib_hi(b8), xv[4 * w + 2], xv[4 * w + 3]);
            }
        } else {
            const uint4 v = lds16(xblk + (uint32_t)(16 * j));
            mma16816_bf16(acc[0], aw[0], bw[0], aw[1], bw[1], v.x, v.y);
            mma16816_bf16(acc[1], aw[2], bw[2], aw[3], bw[3], v.z, v.w);
        }
    }
    return diag_part(acc, lane);
}

// 8 fp16 values of h as bf16 high and low parts, h = high + low exactly (an fp16 value has 11
// significant bits, a bf16 8, and the remainder fits in another bf16): registers 0..3 the high
// parts of the pairs (0, 1) .. (6, 7), 4..7 the low parts.  sum: the values, in fp32.
__device__ __forceinline__ void hilo_from_f16(uint4 v, uint32_t* p, float& sum) {
    const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
        const __nv_bfloat162 hi = __floats2bfloat162_rn(f.x, f.y);
        const float2 fh = __bfloat1622float2(hi);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x - fh.x, f.y - fh.y);
        p[i] = *reinterpret_cast<const uint32_t*>(&hi);
        p[4 + i] = *reinterpret_cast<const uint32_t*>(&lo);
        sum += f.x + f.y;
    }
}

// WK: MOE_W_INT4_ROWSCALE or MOE_W_BF16.  NDK: 16-byte groups of a gate/up row per lane (d / 1024
// for int4, d / 256 for bf16); NF: the same for a down row (f / 1024, f / 256).  NT: tokens (1 or
// 2).  With two tokens the CTA's two halves select for one token each, the routed slots are
// token-major (t k + rank), the shared expert's slots follow (NT k + t), and each shared row pair
// is applied to both tokens from one read.
template <int WK, int NDK, int NF, int NT>
__global__ void __launch_bounds__(kFzMaxThreads, 1) decode_fused_kernel(const FusedArgs a) {
    // [x~ lane blocks][kFzStages][warps][stage]: stage s of every warp is one region; x (plain
    // bf16, 2d bytes) lands in the last stage's region during phase A
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[kFzMaxWarps][kFzStages];
    __shared__ int4 s_desc[kFzMaxWarps][kFzStages];       // gate/up stage: slot, row, scale slots
    __shared__ __align__(8) uint64_t s_xbar;              // x -> shared memory
    __shared__ __align__(8) uint64_t s_rbar;              // the router pieces -> shared memory
    __shared__ float ys[NT * kFzMaxSlots][fz_rows_max(NT)];
    // the routed slots are the chosen experts in rank order (token-major)
    __shared__ const uint8_t* s_gu[NT * kFzMaxSlots];      // their weights (the layer's pointer table)
    __shared__ const float* s_gus[NT * kFzMaxSlots];
    __shared__ const uint8_t* s_dn[NT * kFzMaxSlots];
    __shared__ const float* s_dns[NT * kFzMaxSlots];
    __shared__ float s_w[NT * kFzMaxSlots];                // their gate weights (set during phase C)
    __shared__ int s_asc[NT * kFzMaxSlots];                // slot of the p-th smallest chosen expert
    __shared__ int sel_e[NT * kFzMaxSlots];                // rank order
    __shared__ int cand_e[NT][kFzMaxPer * kFzMaxSlots];   // selection candidates, k per warp
    __shared__ uint2 cand_k[NT][kFzMaxPer * kFzMaxSlots]; // and their keys
    __shared__ double sel_l[NT * kFzMaxSlots];
    __shared__ unsigned long long s_base;                 // arrivals before this launch
    __shared__ int s_ok;

    constexpr bool BF = WK == MOE_W_BF16;
    constexpr int d = 32 * NDK * FzKind<WK>::COLS, f = 32 * NF * FzKind<WK>::COLS;
    constexpr int XR = FzKind<WK>::XR, HR = FzKind<WK>::HR;
    const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
    const int nwc = blockDim.x / kWarp;                    // warps of this CTA
    const int G = gridDim.x;
    const int gw = warp * G + blockIdx.x, nw = G * nwc;    // warp-major: low numbers on every SM
    const int k = a.k, E = a.E;
    constexpr uint32_t gu_row = FzKind<WK>::row_bytes(d), dn_row_b = FzKind<WK>::row_bytes(f);
    constexpr int nst = kFzStages;                         // ring stages per warp
    constexpr int nch = d / 1024;                          // 1024-column router pieces per expert
    constexpr uint32_t stage_bytes = 2 * gu_row + 32;
    // x~ lane blocks: lane L's groups in its visiting order, padded by 16 bytes so that the lanes'
    // 16-byte loads meet no bank conflict
    constexpr uint32_t kLaneBlk = (BF ? 16 : 64) * NDK + 16;
    constexpr uint32_t kXtBytes = (32 * kLaneBlk + 127) / 128 * 128;
    const uint32_t xt_s = saddr(smem);                     // token t's lane blocks at xt_s + t kXtBytes
    const uint32_t rings_s = xt_s + NT * kXtBytes;
    auto st_s = [&](int s) { return rings_s + ((uint32_t)s * nwc + warp) * stage_bytes; };
    auto st_g = [&](int s) { return smem + NT * kXtBytes + ((size_t)s * nwc + warp) * stage_bytes; };
    const uint32_t xraw_s = rings_s + (uint32_t)(nst - 1) * nwc * stage_bytes;   // token t at + 2 d t
    const int n_sh = a.S ? f : 0;                          // shared row pairs (each for every token)
    const int nrs = NT * k;                                // routed slots
    const int n_tasks = n_sh + nrs * f;
    auto count_of = [&](int lo, int hi) {                  // my tasks among [lo, hi)
        const int first = lo + ((gw - lo) % nw + nw) % nw; // smallest t >= lo with t == gw (mod nw)
        return first < hi ? (hi - first + nw - 1) / nw : 0;
    };
    const int my_sh = count_of(0, n_sh);
    const int my_tasks = my_sh + count_of(n_sh, n_tasks);
    // task i of this warp is t = gw + i * nw (shared ones first because gw < nw)
    // this CTA's output rows and the warp's share of the (slot, row) items
    const int j0 = (int)((int64_t)blockIdx.x * d / G), rj = (int)((int64_t)(blockIdx.x + 1) * d / G) - j0;
    const int nslots = nrs + NT * a.S;
    const int n_items = nslots * rj;
    const int it0 = (int)((int64_t)warp * n_items / nwc), it1 = (int)((int64_t)(warp + 1) * n_items / nwc);
    // the lane's segment (g) and quarter (c): byte offsets within a gate/up row and a down row
    const int lg = lane >> 2, lc = lane & 3;
    const uint32_t gu_lane_off = (uint32_t)lg * (gu_row / 8) + (uint32_t)lc * (16 * NDK);
    const uint32_t dn_lane_off = (uint32_t)lg * (dn_row_b / 8) + (uint32_t)lc * (16 * NF);
    const int grot = gu_rot<NDK>(lane), drot = dn_rot<NF>(lane);
    const uint64_t pol_first = policy_evict_first();

    unsigned long long* const trace = a.trace ? a.trace + (size_t)blockIdx.x * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (tid == 0 && trace) trace[i] = now_ns();
    };
    stamp(0);
    if (lane == 0) {
        for (int s = 0; s < nst; ++s) bar_init(saddr(&bars[warp][s]), 1);
        if (warp == 0) {
            bar_init(saddr(&s_xbar), 1);
            bar_init(saddr(&s_rbar), 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        bar_expect_tx(saddr(&s_xbar), 2u * d * NT);
        bulk_g2s(xraw_s, a.x, 2u * d * NT, saddr(&s_xbar));
    }

    // ---- the ring: use q of this warp goes to stage q % nst
    //      q < my_tasks: gate/up row pair (task q); q >= my_tasks: down stage (lane 0's cursor)
    int issued = 0;               // lane 0: next use to issue
    int n_dn = 0;                 // this warp's down stages
    auto sliver = [](const float* p) { return reinterpret_cast<const float*>((uintptr_t)p & ~(uintptr_t)15); };
    // lane 0's cursors: the routed (slot, row) of its next routed row pair, the next down item
    int gu_u = -1, gu_r = 0;
    int dn_u = it0 / max(rj, 1), dn_row = it0 - dn_u * rj, dn_it = it0;
    auto dn_count = [&](int it, int row) { return min(min(a.dn_rows, it1 - it), rj - row); };
    auto issue = [&](int q) {
        const int sidx = q % nst;
        const uint32_t bar = saddr(&bars[warp][sidx]);
        const uint32_t dst = st_s(sidx);
        if (q < my_tasks) {
            const int t = gw + q * nw;
            const uint8_t* rows;
            const float* sc;
            int r, slot;
            if (t < n_sh) {
                rows = a.sh_gate_up + (size_t)t * gu_row;
                sc = a.sh_gu_scale + t;
                r = t;
                slot = nrs;                                // the first shared slot
            } else {
                if (gu_u < 0) {
                    gu_u = (t - n_sh) / f;
                    gu_r = t - n_sh - gu_u * f;
                }
                r = gu_r;
                slot = gu_u;
                rows = s_gu[gu_u] + (size_t)gu_r * gu_row;
                sc = s_gus[gu_u] + gu_r;
                for (gu_r += nw; gu_r >= f; gu_r -= f) ++gu_u;
            }
            // the consumer finds its row and, in the two 16-byte slivers, its two scales
            // bf16 rows have no scales (the slivers are not copied)
            s_desc[warp][sidx] = BF ? make_int4(slot, r, 0, 0)
                                    : make_int4(slot, r, (int)(((uintptr_t)sc >> 2) & 3), 4 + (int)(((uintptr_t)(sc + f) >> 2) & 3));
            bar_expect_tx(bar, BF ? 2 * gu_row : stage_bytes);
            bulk_g2s_hint(dst, rows, gu_row, bar, pol_first);
            bulk_g2s_hint(dst + gu_row, rows + (size_t)f * gu_row, gu_row, bar, pol_first);
            if (!BF) {
                bulk_g2s(dst + 2 * gu_row, sliver(sc), 16, bar);
                bulk_g2s(dst + 2 * gu_row + 16, sliver(sc + f), 16, bar);
            }
        } else {
            const int n = dn_count(dn_it, dn_row);
            const uint8_t* W = dn_u < nrs ? s_dn[dn_u] : a.sh_down;
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
        const bool ok = bar_wait(saddr(&bars[warp][q % nst]), (uint32_t)(q / nst) & 1u);
        __syncwarp();                                      // lane 0's stage descriptor is visible
        return __all_sync(0xffffffffu, ok);
    };
    auto drain = [&](int from) {      // lane 0: let every copy still in flight land
        if (lane == 0)
            for (int q2 = from; q2 < issued; ++q2)
                bar_wait(saddr(&bars[warp][q2 % nst]), (uint32_t)(q2 / nst) & 1u);
    };

    // ---- A: this warp's first router pieces (coalesced loads, all in flight) while x lands; once
    //      x is in, the shared expert's row pairs (they need no routing) go into every stage but
    //      the last, which holds x until x~ is built and the router pieces are done
    int limit = my_sh;            // lane 0: uses that may be issued so far
    const int n_units = E * nch;
    float4 rw[8];
    if (gw < n_units) {
        const int e = gw / nch, p = gw - e * nch;
        load_router_piece(a.router_w + (size_t)e * d + 1024 * p, lane, rw);
    }
    bool ok = __all_sync(0xffffffffu, bar_wait(saddr(&s_xbar), 0u));
    stamp(11);
    if (lane == 0)
        while (issued < my_sh && issued < nst - 1) issue(issued++);
    // the shared expert's down rows of this CTA are read last: start pulling them into L2
    if (a.S && tid == kWarp && rj > 0) prefetch_l2(a.sh_down + (size_t)j0 * dn_row_b, (uint32_t)rj * dn_row_b);
    // x as the lanes' MMA operand, once per CTA: thread t places the 8-column groups t, t + threads,
    // ... into the lane blocks.  int4: fp16 x~ = x 2^sigma, sigma from max|x|, the pairs of
    // pairs_from_bf16; bf16: the bf16 values as they are.  The sum of x~ (fp64) is reduced in a
    // fixed order, so every CTA gets the same value.
    __shared__ float s_redf[kFzMaxWarps];
    __shared__ double s_redd[kFzMaxWarps];
    int sig[NT] = {};
    double xs[NT] = {};           // per token: sum of x~ = x 2^sigma over the whole row (bf16: of x)
#pragma unroll
    for (int tk = 0; tk < NT; ++tk) {
        const uint32_t xr = xraw_s + 2u * d * tk;             // token tk's plain x
        const uint32_t xt = xt_s + kXtBytes * tk;             // and its lane blocks
        if constexpr (BF) {
            float part = 0.0f;
            for (int g = tid; g < d / 8; g += blockDim.x) {
                const uint4 v = lds16(xr + 16u * (uint32_t)g);
                const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) part += __uint_as_float(ws[i] << 16) + __uint_as_float(ws[i] & 0xffff0000u);
                // group g (8 columns) belongs to lane L = 4 seg + quarter, as its group q
                const int seg = g / (d / 64), rem = g - seg * (d / 64);
                const int cq = rem / NDK, q = rem - cq * NDK, L = 4 * seg + cq;
                int j = q - gu_rot<NDK>(L);
                if (j < 0) j += NDK;
                sts16(xt + (uint32_t)L * kLaneBlk + (uint32_t)j * 16u, v);
            }
            const double pd = warp_sum_d((double)part);
            if (lane == 0) s_redd[warp] = pd;
            __syncthreads();
            for (int w = 0; w < nwc; ++w) xs[tk] += s_redd[w];
        } else {
            float m = 0.0f;
            for (int g = tid; g < d / 8; g += blockDim.x) {
                const uint4 v = lds16(xr + 16u * (uint32_t)g);
                const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(ws[i] << 16)), fabsf(__uint_as_float(ws[i] & 0xffff0000u))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) s_redf[warp] = m;
            __syncthreads();
            m = 0.0f;
            for (int w = 0; w < nwc; ++w) m = fmaxf(m, s_redf[w]);
            sig[tk] = scale_exp(m);
            const float s1 = exp2i(sig[tk]), s16 = exp2i(sig[tk] - 4);
            float part = 0.0f;
            for (int g = tid; g < d / 8; g += blockDim.x) {
                uint32_t pr[4];
                pairs_from_bf16(lds16(xr + 16u * (uint32_t)g), s1, s16, pr, part);
                // group g belongs to lane L = 4 seg + quarter, as word w of its group q
                const int seg = g / (d / 64), rem = g - seg * (d / 64);
                const int cq = rem / (4 * NDK), rem2 = rem - cq * (4 * NDK);
                const int q = rem2 >> 2, w = rem2 & 3, L = 4 * seg + cq;
                int j = q - gu_rot<NDK>(L);
                if (j < 0) j += NDK;
                sts16(xt + (uint32_t)L * kLaneBlk + (uint32_t)(4 * j + w) * 16u, make_uint4(pr[0], pr[1], pr[2], pr[3]));
            }
            const double pd = warp_sum_d((double)part);
            if (lane == 0) s_redd[warp] = pd;
            __syncthreads();
            for (int w = 0; w < nwc; ++w) xs[tk] += s_redd[w];
        }
        if (tk + 1 < NT) __syncthreads();                  // s_redf / s_redd are reused
    }
    // router pieces: unit u = (expert u / nch, columns [1024 p, 1024 p + 1024), p = u % nch)
    auto piece = [&](int u, const float4 (&wv)[8]) {
        const int p = u % nch;
#pragma unroll
        for (int tk = 0; tk < NT; ++tk) {                  // one router row piece, every token
            const double v = warp_sum_d(router_piece(wv, xraw_s + 2u * d * tk + 2048u * p, lane));
            if (lane == 0) __stcg(a.rpart + (size_t)tk * n_units + u, v);
        }
    };
    if (gw < n_units) piece(gw, rw);
    for (int u = gw + nw; u < n_units; u += nw) {
        const int e = u / nch, p = u - e * nch;
        load_router_piece(a.router_w + (size_t)e * d + 1024 * p, lane, rw);
        piece(u, rw);
    }
    stamp(1);
    const uint32_t xblk = xt_s + (uint32_t)lane * kLaneBlk;   // this lane's operand block (token 0)
    float xoffs[NT], xunscale[NT];                          // per token: 8 sum x~ 2^-sigma, 2^(24 - sigma)
#pragma unroll
    for (int tk = 0; tk < NT; ++tk) {
        xoffs[tk] = 8.0f * (float)xs[tk] * exp2i(-sig[tk]);
        xunscale[tk] = exp2i(-sig[tk]) * 16777216.0f;
    }
    // selection: the CTA's halves take one token each (NT = 2); thread ltid of half tt holds
    // expert ltid of token tt
    const int nwh = nwc / NT, tt = warp / nwh, lw = warp - tt * nwh, ltid = tid - tt * nwh * kWarp;
    const float my_bias = a.bias && ltid < E ? a.bias[ltid] : 0.0f;
    __syncthreads();                                       // the last stage (x) is free
    if (tid == 0) {                                        // barrier 0: every piece is stored
        const unsigned long long old = arrive(a.bar);
        s_base = old - old % (2ull * G);
    }
    stamp(2);

    // ---- one gate/up row pair: stage of use q.  Lane n of the warp keeps the n-th pending result
    //      (g, u, index into h); every 32 row pairs, and at the end, all lanes finish theirs at once.
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
    // one gate/up row pair (stage of use q): a routed slot's for its token, a shared one's for
    // every token (the row pair decoded from the one copy in shared memory)
    auto gate_up_stage = [&](int q) {
        const int s = q % nst;
        const int4 dsc = s_desc[warp][s];
        const bool sh = dsc.x >= nrs;
        const int t0 = sh ? 0 : dsc.x / k;                 // routed slots are token-major
        const uint32_t ra = st_s(s), rb = ra + gu_row;
        float2 parts[NT];
        parts[0] = rows_mma_x<WK, NDK>(ra, rb, gu_lane_off, grot, xblk + kXtBytes * t0, lane);
#pragma unroll
        for (int tk = 1; tk < NT; ++tk)
            if (sh) parts[tk] = rows_mma_x<WK, NDK>(ra, rb, gu_lane_off, grot, xblk + kXtBytes * tk, lane);
        const float* scs = reinterpret_cast<const float*>(st_g(s) + 2 * gu_row);
        const float sg = BF ? 1.0f : scs[dsc.z], su = BF ? 1.0f : scs[dsc.w];
        __syncwarp();                                      // the stage is free again
        if (lane == 0)
            while (issued < limit && issued < q + 1 + nst) issue(issued++);
#pragma unroll
        for (int tk = 0; tk < NT; ++tk) {
            if (tk > 0 && !sh) break;
            const int tok = sh ? tk : t0;
            const float ag = warp_sum(parts[tk].x), au = warp_sum(parts[tk].y);
            if (lane == n_pend) {
                const float xu = pick_tok(xunscale, tok), xo = pick_tok(xoffs, tok);
                p_g = BF ? ag : sg * fmaf(ag, xu, -xo);
                p_u = BF ? au : su * fmaf(au, xu, -xo);
                p_h = (dsc.x + (sh ? tk : 0)) * f + h_pos<f>(dsc.y);
            }
            if (++n_pend == kWarp) flush();
        }
    };

    int q = 0;                    // next use to consume
    for (; ok && q < my_sh; ++q) {                         // the shared expert's row pairs
        if (lane == 0)
            while (issued < limit && issued < q + nst) issue(issued++);
        if (!wait_use(q)) { ok = false; break; }
        gate_up_stage(q);
    }

    // ---- B: selection by the whole CTA once every piece of the logits is stored.  The rings are
    //      idle: the router pieces, then the keys and logits, go to their start.
    __syncthreads();
    stamp(3);
    const uint32_t rbytes = ((uint32_t)(NT * n_units) * 8u + 15u) & ~15u;
    uint8_t* const rings = smem + NT * kXtBytes;           // generic address of rings_s
    uint2* keys = reinterpret_cast<uint2*>(rings + rbytes);    // [NT][E] keys, order-preserving integers
    double* lgs = reinterpret_cast<double*>(keys + NT * E);    // [NT][E] logits
    if (tid == 0) {
        const bool bok = wait_arrivals(a.bar, s_base + (unsigned long long)G);
        if (!bok) {
            latch_status(a.status, MOE_ERR_TIMEOUT);
        } else {
            bar_expect_tx(saddr(&s_rbar), rbytes);
            bulk_g2s(rings_s, a.rpart, rbytes, saddr(&s_rbar));
        }
        s_ok = bok;
    }
    __syncthreads();
    stamp(4);
    bool sel = s_ok != 0;
    if (sel) {
        const bool landed = bar_wait(saddr(&s_rbar), 0u);
        if (landed && tt < NT && ltid < E) {
            const double* rp = reinterpret_cast<const double*>(rings) + (size_t)tt * n_units;
            double l = 0.0;
            for (int p = 0; p < nch; ++p) l += rp[ltid * nch + p];
            lgs[tt * E + ltid] = l;
            // key -> unsigned 64-bit integer of the same order (-0 folded into +0; NaN is -inf)
            const long long b = __double_as_longlong(topk_key(l, my_bias, a.router) + 0.0);
            const unsigned long long o = b < 0 ? ~(unsigned long long)b : (unsigned long long)b | (1ull << 63);
            keys[tt * E + ltid] = make_uint2((uint32_t)(o >> 32), (uint32_t)o);
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
        const int nwe = (E + kWarp - 1) / kWarp;           // warps holding experts (per half)
        if (sel && tt < NT && lw < nwe) {
            const int e = ltid;
            const uint2 mk = e < E ? keys[tt * E + e] : make_uint2(0u, 0u);   // below every real key
            int rank = 0;
#pragma unroll 4
            for (int o = 1; o < kWarp; ++o) {
                const int jl = (lane + o) & (kWarp - 1);
                const uint2 kj = make_uint2(__shfl_sync(0xffffffffu, mk.x, jl), __shfl_sync(0xffffffffu, mk.y, jl));
                rank += beats(kj, lw * kWarp + jl, mk, e) ? 1 : 0;
            }
            if (lane < k) {
                cand_e[tt][lw * k + lane] = -1;
                cand_k[tt][lw * k + lane] = make_uint2(0u, 0u);
            }
            __syncwarp();
            if (e < E && rank < k) {
                cand_e[tt][lw * k + rank] = e;
                cand_k[tt][lw * k + rank] = mk;
            }
        }
        __syncthreads();
        stamp(12);
        const int nc = nwe * k;                            // candidate slots per token
        if (sel && tt < NT && ltid < nc) {
            const int e = cand_e[tt][ltid];
            if (e >= 0) {
                // the candidate's weight pointers: loaded while the rank is counted
                const void* pw[4] = {ex_gate_up(a.etab, E, e), ex_gu_scale(a.etab, E, e), ex_down(a.etab, E, e),
                                     ex_dn_scale(a.etab, E, e)};
                const uint2 mk = cand_k[tt][ltid];
                int rank = 0;
#pragma unroll 8
                for (int c = 0; c < nc; ++c)               // empty slots hold key 0, below every real key
                    rank += beats(cand_k[tt][c], cand_e[tt][c], mk, e) ? 1 : 0;
                if (rank < k) {
                    const int slot = tt * k + rank;
                    sel_e[slot] = e;
                    sel_l[slot] = lgs[tt * E + e];
                    s_gu[slot] = static_cast<const uint8_t*>(pw[0]);
                    s_gus[slot] = static_cast<const float*>(pw[1]);
                    s_dn[slot] = static_cast<const uint8_t*>(pw[2]);
                    s_dns[slot] = static_cast<const float*>(pw[3]);
                }
            }
        }
        __syncthreads();
        stamp(13);
    }
    stamp(14);
    // the keys were written through the generic proxy; TMA writes into the same bytes come next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    stamp(15);
    __syncthreads();              // the slots' pointers are set; the rings may be used again
    stamp(6);
    const bool routed = sel;

    // the scales of this warp's down items (slot, row), lane i holding item it0 + 32 r + i
    float dsc_r[kFzScRegs];
#pragma unroll
    for (int r = 0; r < kFzScRegs; ++r) {
        const int it = it0 + kWarp * r + lane;
        float v = 0.0f;
        if (routed && it < it1) {
            const int u = it / rj, row = it - u * rj;
            v = BF ? 1.0f : __ldg((u < nrs ? s_dns[u] : a.sh_dn_scale) + j0 + row);
        }
        dsc_r[r] = v;
    }

    // ---- C: the routed row pairs; then the first down stages (independent of h)
    for (int it = it0, row = it0 - (it0 / max(rj, 1)) * rj; it < it1; ++n_dn) {
        const int n = dn_count(it, row);
        it += n;
        row = row + n == rj ? 0 : row + n;
    }
    if (ok && routed) {
        limit = my_tasks + n_dn;
        if (lw == 0 && tt < NT) {
            // the gate weights are needed only by the combine: the first warp of each half
            // computes its token's here, with its first routed rows already in flight, instead of
            // on the way into this phase
            if (lane == 0)
                while (issued < limit && issued < q + nst) issue(issued++);
            const int sb = tt * k;                         // the token's first slot
            const TopkPick pk = topk_finish(lane < k ? sel_e[sb + lane] : -1, lane < k ? sel_l[sb + lane] : 0.0, k,
                                            a.router, a.scaling, lane);
            if (lane < k) {
                s_w[sb + lane] = pk.w;
                s_asc[sb + pk.pos] = sb + lane;
                if (blockIdx.x == 0) {
                    a.idx[sb + lane] = pk.e;
                    a.wts[sb + lane] = pk.w;
                    a.asc[sb + pk.pos] = lane;
                    if (NT == 1) a.ulist[pk.pos] = pk.e;
                }
            }
            if (blockIdx.x == 0 && lane == 0) {
                if (NT == 1) *a.n_unique = k;
                a.xsum[tt] = pick_tok(xs, tt) * (double)exp2i(-pick_tok(sig, tt));
            }
        }
        for (; q < my_tasks; ++q) {
            if (lane == 0)
                while (issued < limit && issued < q + nst) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            gate_up_stage(q);
        }
        if (ok && lane == 0)
            while (issued < limit && issued < q + nst) issue(issued++);
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

    // ---- D: down rows of this CTA's output block, slot by slot, two rows per MMA
    if (ok && s_ok) {
        uint32_t hr[NF][HR];
        float hoff = 0.0f, hun = 0.0f;                     // 8 sum h~, 2^(24 - tau) of the current slot
        int cu = it0 / max(rj, 1), crow = it0 - cu * rj, hu = -1;
        for (int it = it0; it < it1; ++q) {
            const int n = dn_count(it, crow);
            if (cu != hu && BF) {                          // bf16: h as exact high + low bf16 parts
                float part = 0.0f;
#pragma unroll
                for (int j = 0; j < NF; ++j) {
                    int qq = j + drot;
                    if (qq >= NF) qq -= NF;
                    const uint4 v = ld_cg16(a.h + (size_t)cu * f + 8 * (qq * kWarp + lane));
                    hilo_from_f16(v, &hr[j][0], part);
                }
                hoff = 0.0f;
                hun = 1.0f;                                // the formula below then gives v itself
                hu = cu;
            } else if (cu != hu) {                         // int4: this slot's h~ (written by other CTAs)
                uint4 hv[NF][4];
                float m = 0.0f;
#pragma unroll
                for (int j = 0; j < NF; ++j) {
                    int qq = j + drot;
                    if (qq >= NF) qq -= NF;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        hv[j][w] = ld_cg16(a.h + (size_t)cu * f + 8 * ((4 * qq + w) * kWarp + lane));
                        const uint32_t ws[4] = {hv[j][w].x, hv[j][w].y, hv[j][w].z, hv[j][w].w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
                            m = fmaxf(m, fmaxf(fabsf(hf.x), fabsf(hf.y)));
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const int tau = scale_exp(m);
                const float s1 = exp2i(tau), s16 = exp2i(tau - 4);
                float part = 0.0f;
                if constexpr (!BF) {
#pragma unroll
                    for (int j = 0; j < NF; ++j)
#pragma unroll
                        for (int w = 0; w < 4; ++w) pairs_from_f16(hv[j][w], s1, s16, &hr[j][4 * w], part);
                }
                hoff = 8.0f * warp_sum(part);
                hun = exp2i(-tau) * 16777216.0f;
                hu = cu;
            }
            if (lane == 0)
                while (issued < limit && issued < q + nst) issue(issued++);
            if (!wait_use(q)) { ok = false; break; }
            const uint32_t st = st_s(q % nst);
#pragma unroll 1
            for (int rr = 0; rr < n; rr += 2) {
                const uint32_t rowA = st + (uint32_t)rr * dn_row_b;
                const uint32_t rowB = rr + 1 < n ? rowA + dn_row_b : rowA;
                const float2 pr = rows_mma<WK, NF, HR, BF>(rowA, rowB, dn_lane_off, drot, hr, lane);
                const float vA = warp_sum(pr.x), vB = warp_sum(pr.y);
                const int iA = it + rr - it0, iB = iA + 1;
                const float sA = __shfl_sync(0xffffffffu, dsc_r[0], iA & 31);
                const float sA1 = __shfl_sync(0xffffffffu, dsc_r[1], iA & 31);
                const float sA2 = __shfl_sync(0xffffffffu, dsc_r[2], iA & 31);
                const float sB = __shfl_sync(0xffffffffu, dsc_r[0], iB & 31);
                const float sB1 = __shfl_sync(0xffffffffu, dsc_r[1], iB & 31);
                const float sB2 = __shfl_sync(0xffffffffu, dsc_r[2], iB & 31);
                const float scA = iA < 32 ? sA : iA < 64 ? sA1 : sA2;
                const float scB = iB < 32 ? sB : iB < 64 ? sB1 : sB2;
                if (lane == 0) {
                    ys[cu][crow + rr] = scA * fmaf(vA, hun, -hoff * hun * (1.0f / 16777216.0f));
                    if (rr + 1 < n) ys[cu][crow + rr + 1] = scB * fmaf(vB, hun, -hoff * hun * (1.0f / 16777216.0f));
                }
            }
            __syncwarp();
            if (lane == 0)
                while (issued < limit && issued < q + 1 + nst) issue(issued++);
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
        for (int it2 = tid; it2 < NT * rj; it2 += blockDim.x) {
            const int tk = it2 / rj, i = it2 - tk * rj;
            float o = 0.0f;
            for (int p = 0; p < k; ++p) {              // ascending expert order
                const int u = s_asc[tk * k + p];
                o = fmaf(s_w[u], ys[u][i], o);
            }
            if (a.S) o += ys[nrs + tk][i];
            const size_t at = (size_t)tk * d + j0 + i;
            if (a.out_bf16)
                static_cast<__nv_bfloat16*>(a.out)[at] = __float2bfloat16_rn(o);
            else
                static_cast<float*>(a.out)[at] = o;
        }
    }
    stamp(10);
}

bool fz_bf16(const LayerDims& L) { return L.wkind == MOE_W_BF16; }
size_t fz_row_bytes(const LayerDims& L, int cols) { return fz_bf16(L) ? (size_t)cols * 2 : (size_t)cols / 2; }
size_t fz_stage_bytes(const LayerDims& L) { return 2 * fz_row_bytes(L, L.d) + 32; }
// Bytes of the x~ lane blocks (the kernel's kXtBytes).
size_t fz_xt_bytes(const LayerDims& L) {
    const size_t blk = fz_bf16(L) ? 16 * (size_t)(L.d / 256) + 16 : 64 * (size_t)(L.d / 1024) + 16;
    return (32 * blk + 127) / 128 * 128;
}
// Warps per CTA: as many (up to 16; an even number for two tokens, whose selection takes one half
// each) as kFzStages ring stages each fit in shared memory beside the tokens' lane blocks.
int fz_warps(const LayerDims& L, int nt) {
    const size_t room = kSmemLimit - fz_static_reserve(nt) - (size_t)nt * fz_xt_bytes(L);
    int w = (int)(room / ((size_t)kFzStages * fz_stage_bytes(L)));
    if (w > kFzMaxWarps) w = kFzMaxWarps;
    return nt > 1 ? w - w % nt : w;
}
size_t fz_dyn_smem(const LayerDims& L, int nt) {
    return (size_t)nt * fz_xt_bytes(L) + (size_t)kFzStages * fz_warps(L, nt) * fz_stage_bytes(L);
}
int fz_dn_rows(const LayerDims& L) {
    const int r = (int)(fz_stage_bytes(L) / fz_row_bytes(L, L.f));
    return r > kFzDnRowsMax ? kFzDnRowsMax : r;
}

template <int NDK, int NT>
const void* fz_pick_f(int nf) {
    return nf == 1 ? (const void*)decode_fused_kernel<MOE_W_INT4_ROWSCALE, NDK, 1, NT>
                   : (const void*)decode_fused_kernel<MOE_W_INT4_ROWSCALE, NDK, 2, NT>;
}
template <int NT>
const void* fz_pick_int4(const LayerDims& L) {
    const int nf = L.f / 1024;
    switch (L.d / 1024) {
        case 1: return fz_pick_f<1, NT>(nf);
        case 2: return fz_pick_f<2, NT>(nf);
        case 3: return fz_pick_f<3, NT>(nf);
        case 4: return fz_pick_f<4, NT>(nf);
        case 5: return fz_pick_f<5, NT>(nf);
        case 6: return fz_pick_f<6, NT>(nf);
        case 7: return fz_pick_f<7, NT>(nf);
        default: return fz_pick_f<8, NT>(nf);
    }
}
const void* fz_pick(const LayerDims& L, int nt) {
    if (fz_bf16(L)) {     // one token; d = 1024 or 2048 (4 or 8 groups), f = 512 or 1024 (2 or 4 groups)
        if (L.d == 1024)
            return L.f == 512 ? (const void*)decode_fused_kernel<MOE_W_BF16, 4, 2, 1>
                              : (const void*)decode_fused_kernel<MOE_W_BF16, 4, 4, 1>;
        return L.f == 512 ? (const void*)decode_fused_kernel<MOE_W_BF16, 8, 2, 1>
                          : (const void*)decode_fused_kernel<MOE_W_BF16, 8, 4, 1>;
    }
    return nt == 2 ? fz_pick_int4<2>(L) : fz_pick_int4<1>(L);
}

}  // namespace

bool decode_fused_shape_ok(const LayerDims& L, int nt) {
    const bool int4_shape = L.wkind == MOE_W_INT4_ROWSCALE && L.d % 1024 == 0 && L.d / 1024 >= 1 && L.d / 1024 <= 8 &&
                            (L.f == 1024 || L.f == 2048);
    const bool bf16_shape = nt == 1 && L.wkind == MOE_W_BF16 && (L.d == 1024 || L.d == 2048) &&
                            (L.f == 512 || L.f == 1024);
    if (nt < 1 || nt > 2) return false;
    if (!((int4_shape || bf16_shape) && (!L.S || L.f_shared == L.f) && L.k + L.S <= kFzMaxSlots &&
          L.E <= kWarp * kFzMaxPer && L.k <= L.E && fz_dn_rows(L) >= 1 && fz_warps(L, nt) >= 4))
        return false;
    // the selection keeps the router pieces, keys and logits in the (idle) rings; each token's
    // experts fit one thread each in its half of the CTA
    const size_t rings = (size_t)kFzStages * fz_warps(L, nt) * fz_stage_bytes(L);
    const size_t sel_bytes = ((size_t)nt * L.E * (L.d / 1024) * 8 + 15) / 16 * 16 + 16 * (size_t)nt * L.E;
    return sel_bytes <= rings && L.E <= fz_warps(L, nt) / nt * kWarp;
}

cudaError_t prepare_decode_fused(const LayerDims& L, int num_sms, bool* usable, int nt) {
    *usable = false;
    if (!decode_fused_shape_ok(L, nt) || (L.d + num_sms - 1) / num_sms > fz_rows_max(nt) || num_sms > kTraceCtas)
        return cudaSuccess;
    // the down items of one warp must fit the scale registers
    const int rows = (L.d + num_sms - 1) / num_sms;
    if (nt * (L.k + L.S) * rows > fz_warps(L, nt) * (kWarp * kFzScRegs - 1)) return cudaSuccess;
    int dev = 0, coop = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess || !coop) return e;
    const void* fn = fz_pick(L, nt);
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    if (fa.sharedSizeBytes > fz_static_reserve(nt)) return cudaSuccess;
    const size_t dyn = fz_dyn_smem(L, nt);
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(kSmemLimit - fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
    int blocks = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, fz_warps(L, nt) * kWarp, dyn);
    if (e != cudaSuccess) return e;
    *usable = blocks >= 1;
    return cudaSuccess;
}

cudaError_t launch_decode_fused(const LayerDims& L, const moe_weights& W, const uint16_t* x, const Workspace& ws,
                                void* out, int num_sms, const Launch& ctx, int nt) {
    FusedArgs a;
    a.router_w = W.router_w;
    a.bias = L.router == MOE_ROUTER_SIGMOID_BIAS ? W.router_bias : nullptr;
    a.x = x;
    a.sh_gate_up = (const uint8_t*)W.shared_gate_up;
    a.sh_gu_scale = W.shared_gate_up_scale;
    a.sh_down = (const uint8_t*)W.shared_down;
    a.sh_dn_scale = W.shared_down_scale;
    a.etab = (const void* const*)ws.etab;
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
    a.trace = L.phase_trace ? ws.trace : nullptr;
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);
    cfg.blockDim = dim3((unsigned)(fz_warps(L, nt) * kWarp));
    cfg.dynamicSmemBytes = fz_dyn_smem(L, nt);
    cfg.stream = ctx.s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&a};
    prof_mark(ctx.prof, MOE_KERNEL_FUSED, true, ctx.s);
    cudaError_t e = cudaLaunchKernelExC(&cfg, fz_pick(L, nt), args);
    prof_mark(ctx.prof, MOE_KERNEL_FUSED, false, ctx.s);
    if (e != cudaSuccess) return e;
    ++*ctx.launches;
    return cudaSuccess;
}

}  // namespace qe
