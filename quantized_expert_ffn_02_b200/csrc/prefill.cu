// prefill.cu -- K5: the batch-union expert FFN as grouped GEMMs on the 5th-generation tensor
// cores (tcgen05), for batches large enough that the expert FFN is a dense contraction.
//
// Prior art on the iliria page ("What's implemented": Metal prefill GEMMs; grouped CPU MoE with
// a ragged descriptor over expert slabs, gate+up fused over one activation).  Here, per unique
// expert and per block of at most 128 of its tokens ("group"):
//
//   GEMM-1  D[r][n] = sum_k Wgu[r][k] * x[n][k] for the 128 gate rows and the matching 128 up
//           rows of one tile, two fp32 accumulators in tensor memory (TMEM); epilogue
//           h = silu(s_g * g) * (s_u * u) -> fp16.
//   GEMM-2  D[j][n] = sum_r Wd[j][r] * h[n][r]; epilogue y = s_d * D -> fp32 per slot.
//
// Weights are the M side (128 rows per tile) and tokens the N side (at most 128, rounded up to
// 16 per group), so a skinny bucket costs little.  The int4 codes are dequantised on use: TMA
// brings the packed rows into shared memory, four converter warps turn each row's nibbles into
// exact 16-bit integers (bf16 for GEMM-1, whose B operand is bf16 x; fp16 for GEMM-2, whose B
// operand is fp16 h) and store them straight into TMEM, where tcgen05.mma reads its A operand;
// B comes from shared memory (TMA, 128-byte swizzle).  The per-row scale is applied in the
// epilogue, so the MMA sees q exactly.
//
// K order.  The nibble trick produces the pair (column i, column i+4) of every 8 columns in one
// 32-bit register; the A operand in TMEM holds two consecutive K elements per column.  So K is
// permuted within each group of 8 as [0,4,1,5,2,6,3,7] on both sides: the gather kernel writes x
// in that order and the GEMM-1 epilogue writes h in that order.  A dot product does not depend
// on the order of its terms.
//
// Roles (640 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer of the packed A rows                 smem ring of 128 KB (16 or 32 stages)
//   warp 18    TMA producer of the B tiles (a box of 16, 32, 64 smem ring of kBStages
//              or 128 rows: the group's tokens rounded up)
//   warp 1     TMEM allocator and MMA issuer 0                    TMEM A ring of kAStages
//   warp 19    the second MMA issuer: GEMM-1 issues the gate rows' MMAs from warp 1 and the up
//              rows' from warp 19, each into its own accumulator (one issuing thread alone is a
//              bottleneck: a tcgen05.mma adding into the result of the one before waits for
//              it); GEMM-2 issues from warp 1 alone and leaves warp 19 idle
//   warps 2-17 converters (A rows -> TMEM), then the epilogue    thread <-> TMEM lane; four sets
//              of four (one warp per TMEM lane quarter each) take every fourth K step, so a
//              set has four MMA steps to hide its TMEM store, and every fourth 16-column block
//              of the epilogue
// Every wait is bounded (2 s by default; the layer option MOE_OPT_WAIT_LIMIT_US sets it); on
// expiry the CTA latches MOE_ERR_TIMEOUT, drains what it issued, frees its TMEM and returns.
#include "internal.cuh"

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

namespace qe {

struct Group {
    int e;        // expert, or -1 for the shared expert
    int slot0;    // first slot (row of xg / h / Y)
    int n;        // tokens in this group (1..128)
    int pad;
};

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 64;
constexpr int kBStages = 4;                           // B tiles (x or h, from L2) in shared memory
constexpr uint32_t kASmBytes = 128 * 1024;            // packed A tiles (from HBM) in shared memory
constexpr int kASmStagesMax = 32;
constexpr int kAStages = 4;                           // converted A tiles in TMEM
constexpr int kConvSets = 4;                          // converter warp sets, one K step in kConvSets each
constexpr int kConvWarps = 4 * kConvSets;             // one warp per TMEM lane quarter per set
constexpr int kBWarp = 2 + kConvWarps;                // the B producer
constexpr int kMaxIssuers = 2;                        // MMA-issuing warps: 1 and kBWarp + 1
constexpr int kGemmThreads = (kBWarp + kMaxIssuers) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kPackedTile = BM * BK / 2;         // 4 KB of packed int4 per 128 x 64 tile
constexpr uint32_t kBTile = BN * BK * 2;              // 16 KB of bf16 / fp16

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase.  Gives up when another role has aborted, or after
// limit_ns (then it latches the timeout and raises the CTA's abort flag).
__device__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status, uint64_t limit_ns) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 63) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort_flag = 1;
                latch_status(status, MOE_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
// Bounded wait used while draining (ignores the abort flag).
__device__ bool wait_bar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try(bar, parity))
        if (globaltimer() - t0 > limit_ns) return false;
    return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma_f16(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
    d |= (uint64_t)1 << 16;                          // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                          // descriptor version
    d |= (uint64_t)2 << 61;                          // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, A and B both bf16 (or both fp16),
// both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16(int n, bool bf16) {
    const uint32_t fmt = bf16 ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// 8 int4 codes of one word -> four registers holding the codes of columns (i, i+4) as a pair of
// 16-bit floats.
//   GEMM-1 (bf16): the nibble goes to the top four mantissa bits of a bf16 1.0, so the pair reads
//     1 + (n ^ 8) / 16 = 3/2 + s/16 exactly (one shift and one LOP3 per pair); the epilogue takes
//     sum s x = 16 D - 24 sum x back out of the accumulator D, with sum x per slot from the gather.
//   GEMM-2 (fp16): magic | (nibble ^ 8) is 1032 + s, and one packed subtraction of the magic leaves
//     s exactly.
template <bool BF16>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t* out) {
    if (BF16) {
        const uint32_t src[4] = {w << 3, w >> 1, w >> 5, w >> 9};   // nibble pair i -> bits 3..6, 19..22
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = lop_sel_xor(src[i], 0x00780078u, 0x3FC03FC0u);
    } else {
        constexpr uint32_t kMask = 0x000F000Fu;
        constexpr uint32_t kMagic = 0x64086408u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t p = lop_sel_xor(w >> (4 * i), kMask, kMagic);
            uint32_t s;
            asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(s) : "r"(p), "r"(kMagic));
            out[i] = s;
        }
    }
}

// Position of f-index r in the K order of GEMM-2 (pairs (i, i+4) of every 8 adjacent).
__device__ __forceinline__ int kperm_pos(int r) {
    const int i = r & 7;
    return (r & ~7) | (i < 4 ? 2 * i : 2 * (i - 4) + 1);
}

struct Tile {
    int a_row0, a_row1;       // first A row (gate / single) and up row, in the A tensor map
    bool shared;
    int ksteps;
    int slot0, n;             // B rows and valid tokens
    int m0;                   // first output row of the tile (f index for GEMM-1, j for GEMM-2)
    const float* sc0;         // scales of a_row0.. (and of a_row1.. for GEMM-1)
    const float* sc1;
};

struct GemmArgs {
    const Group* groups;
    const int* n_groups;      // [0] routed groups, [1] shared groups
    const float* scale;       // routed experts: [E][rows_e]
    const float* scale_sh;    // shared expert: [rows_sh]
    int rows_e;               // A rows per routed expert (2f or d)
    int f, f_sh;              // gate/up: output rows of routed / shared experts; down: unused
    int mt_r, mt_s;           // M tiles per routed / shared group
    int k_r, k_s;             // K of routed / shared GEMMs
    int ld_out;               // h row stride (fmax) or Y row stride (d)
    void* out;                // h (fp16 bits) or Y (fp32)
    int* status;
    const float* xsum_slot;   // gate/up: sum of x of each slot's token
    uint64_t wait_ns;         // limit of every bounded wait
    int skip_b;               // test hook: the B producer issues no copies (the MMA's wait runs out)
};

template <bool GATED>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, int t, int nr) {
    Tile tl;
    int g, m;
    const int routed_tiles = nr * a.mt_r;
    if (t < routed_tiles) {
        g = t / a.mt_r;
        m = t % a.mt_r;
        tl.shared = false;
    } else {
        const int t2 = t - routed_tiles;
        g = nr + t2 / a.mt_s;
        m = t2 % a.mt_s;
        tl.shared = true;
    }
    const Group gr = a.groups[g];
    tl.slot0 = gr.slot0;
    tl.n = gr.n;
    tl.m0 = m * BM;
    if (GATED) {
        const int f = tl.shared ? a.f_sh : a.f;
        const int base = tl.shared ? 0 : gr.e * a.rows_e;
        tl.a_row0 = base + tl.m0;
        tl.a_row1 = base + f + tl.m0;
        const float* sc = tl.shared ? a.scale_sh : a.scale + (size_t)gr.e * a.rows_e;
        tl.sc0 = sc + tl.m0;
        tl.sc1 = sc + f + tl.m0;
        tl.ksteps = a.k_r / BK;
    } else {
        const int base = tl.shared ? 0 : gr.e * a.rows_e;
        tl.a_row0 = base + tl.m0;
        tl.a_row1 = 0;
        const float* sc = tl.shared ? a.scale_sh : a.scale + (size_t)gr.e * a.rows_e;
        tl.sc0 = sc + tl.m0;
        tl.sc1 = nullptr;
        tl.ksteps = (tl.shared ? a.k_s : a.k_r) / BK;
    }
    return tl;
}

template <bool GATED>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA_sh,
            const __grid_constant__ CUtensorMap tmB16, const __grid_constant__ CUtensorMap tmB32,
            const __grid_constant__ CUtensorMap tmB64, const __grid_constant__ CUtensorMap tmB128,
            const GemmArgs args) {
    constexpr int NA = GATED ? 2 : 1;                     // A tiles per stage
    // MMA issuers.  A tcgen05.mma waits for the one before it from the same thread when both add
    // into one accumulator, and one thread issues no faster than about one per 36 ns however
    // independent its MMAs; several issuing warps, each with its own accumulator, share the
    // tensor pipe instead.  GEMM-1: one warp for the gate rows, one for the up rows (measured
    // 7 % faster than one warp for both).  GEMM-2 keeps one issuer: three warps dealing its K
    // steps into three accumulators measured 37 % slower (0.58 against 0.38 us per K step).
    constexpr int NI = GATED ? 2 : 1;
    // The packed weights stream from HBM and need many bytes in flight; B comes from L2.  So A and
    // B have rings of their own, A's much deeper.
    constexpr int kSA = (int)(kASmBytes / (NA * kPackedTile));   // A stages: 16 (gate/up) or 32
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned working area: B tiles first (swizzle atoms), then packed A tiles
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sB = base;                             // kBStages x 16 KB
    const uint32_t sA = base + kBStages * kBTile;         // kSA x NA x 4 KB
    __shared__ __align__(8) uint64_t bars[2 * kASmStagesMax + 2 * kBStages + 2 * kAStages + 3];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int consumed_sh[kConvWarps];               // A stages consumed by each converter warp
    __shared__ int issued_sh;                             // A stages issued
    __shared__ int b_issued_sh, b_consumed_sh;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };                       // A landed (smem)
    auto empty_bar = [&](int s) { return bar0 + 8u * (kSA + s); };              // A converted
    auto bfull_bar = [&](int s) { return bar0 + 8u * (2 * kSA + s); };          // B landed
    auto bempty_bar = [&](int s) { return bar0 + 8u * (2 * kSA + kBStages + s); };   // B consumed
    auto afull_bar = [&](int s) { return bar0 + 8u * (2 * kSA + 2 * kBStages + s); };  // A in TMEM
    auto aempty_bar = [&](int s) { return bar0 + 8u * (2 * kSA + 2 * kBStages + kAStages + s); };
    const uint32_t accfull_bar = bar0 + 8u * (2 * kSA + 2 * kBStages + 2 * kAStages);
    const uint32_t accempty_bar = accfull_bar + 8u;
    const uint32_t final_bar = accfull_bar + 16u;

    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSA; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 4);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(bfull_bar(s), 1);
            mbar_init(bempty_bar(s), NI);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(afull_bar(s), 4);
            mbar_init(aempty_bar(s), NI);
        }
        mbar_init(accfull_bar, NI);
        mbar_init(accempty_bar, kConvWarps);
        mbar_init(final_bar, NI);
        abort_flag = 0;
        issued_sh = 0;
        b_issued_sh = 0;
        b_consumed_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    // TMEM columns: the accumulators (GEMM-1: gate [0, 128), up [128, 256); GEMM-2: one per
    // issuer), then the A ring.
    const uint32_t acc0 = tmem, acc1 = tmem + BN, acc2 = tmem + 2 * BN;
    const uint32_t a_ring = tmem + (GATED ? 2 * BN : NI * BN);
    constexpr uint32_t kAStageCols = NA * (BK / 2);       // 32 columns per 128 x 64 A tile

    const int nr = args.n_groups[0], ns = args.n_groups[1];
    const int n_tiles = nr * args.mt_r + ns * args.mt_s;
    volatile int* abortp = &abort_flag;
    int* status = args.status;
    const uint64_t lim = args.wait_ns;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int ks = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const Tile tl = decode_tile<GATED>(args, t, nr);
                const CUtensorMap* mapA = tl.shared ? &tmA_sh : &tmA;
                for (int kk = 0; kk < tl.ksteps; ++kk, ++ks) {
                    const int s = ks % kSA;
                    if (!(ok = wait_bar(empty_bar(s), ((ks / kSA) & 1) ^ 1, abortp, status, lim))) break;
                    mbar_expect_tx(full_bar(s), NA * kPackedTile);
                    tma_load_2d(sA + s * NA * kPackedTile, mapA, full_bar(s), kk * (BK / 2), tl.a_row0);
                    if (GATED) tma_load_2d(sA + s * NA * kPackedTile + kPackedTile, mapA, full_bar(s), kk * (BK / 2),
                                           tl.a_row1);
                }
            }
            issued_sh = ks;
        }
    } else if (warp == 1 || (warp > kBWarp && warp - kBWarp < NI)) {
        // ------------------------------------------------------------------ MMA issuers
        const int ii = warp == 1 ? 0 : warp - kBWarp;      // issuer index
        const uint32_t my_acc = tmem + (uint32_t)ii * BN;
        if (lane == 0) {
            int ks = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
                const Tile tl = decode_tile<GATED>(args, t, nr);
                const int nmma = (tl.n + 15) & ~15;
                const uint32_t idesc = idesc_f16(nmma, GATED);
                if (!(ok = wait_bar(accempty_bar, (tc & 1) ^ 1, abortp, status, lim))) break;
                tc_fence_after();
                for (int kk = 0; kk < tl.ksteps; ++kk, ++ks) {
                    const int s = ks % kBStages, sa = ks % kAStages;
                    if (!(ok = wait_bar(bfull_bar(s), (ks / kBStages) & 1, abortp, status, lim))) break;
                    if (!(ok = wait_bar(afull_bar(sa), (ks / kAStages) & 1, abortp, status, lim))) break;
                    tc_fence_after();
                    const uint64_t bdesc = sw128_desc(sB + s * kBTile);
                    const uint32_t a0 = a_ring + sa * kAStageCols;
#pragma unroll
                    for (int j = 0; j < BK / 16; ++j) {
                        if (GATED) {               // issuer 0: the gate rows, issuer 1: the up rows
                            mma_f16(my_acc, a0 + (uint32_t)ii * (BK / 2) + 8 * j, bdesc + 2 * j, idesc, (kk | j) != 0);
                        } else {
                            const int u = (BK / 16) * kk + j;          // the tile's u-th MMA
                            if (u % NI == ii) mma_f16(my_acc, a0 + 8 * j, bdesc + 2 * j, idesc, u >= NI);
                        }
                    }
                    mma_commit(bempty_bar(s));
                    mma_commit(aempty_bar(sa));
                }
                if (ok) mma_commit(accfull_bar);
            }
            if (ii == 0) b_consumed_sh = ks;
            // drain: every MMA issued so far completes before TMEM is released
            mma_commit(final_bar);
            wait_bar_drain(final_bar, 0, lim);
        }
        __syncwarp();
    } else if (warp == kBWarp) {
        // ------------------------------------------------------------------ TMA producer of B
        if (lane == 0) {
            int ks = 0;
            bool ok = !args.skip_b;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const Tile tl = decode_tile<GATED>(args, t, nr);
                // the smallest box that holds the group's tokens (rows past them are not read)
                const int nbox = tl.n <= 16 ? 16 : tl.n <= 32 ? 32 : tl.n <= 64 ? 64 : 128;
                const CUtensorMap* mapB = nbox == 16 ? &tmB16 : nbox == 32 ? &tmB32 : nbox == 64 ? &tmB64 : &tmB128;
                for (int kk = 0; kk < tl.ksteps; ++kk, ++ks) {
                    const int s = ks % kBStages;
                    if (!(ok = wait_bar(bempty_bar(s), ((ks / kBStages) & 1) ^ 1, abortp, status, lim))) break;
                    mbar_expect_tx(bfull_bar(s), (uint32_t)nbox * BK * 2u);
                    tma_load_2d(sB + s * kBTile, mapB, bfull_bar(s), kk * BK, tl.slot0);
                }
            }
            b_issued_sh = ks;
        }
        __syncwarp();
    } else if (warp > kBWarp) {
        // an issuer warp this GEMM does not use: nothing to do
    } else {
        // ------------------------------------------------------------------ converters + epilogue
        const int q = warp & 3;                            // TMEM lane quarter of this warp
        const int set = (warp - 2) / 4;                    // K steps with ks % kConvSets == set
        const int r = 32 * q + lane;                       // tile row owned by this thread
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        int ks = 0, tc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
            const Tile tl = decode_tile<GATED>(args, t, nr);
            for (int kk = 0; kk < tl.ksteps; ++kk, ++ks) {
                if (ks % kConvSets != set) continue;
                const int s = ks % kSA, sa = ks % kAStages;
                ok = wait_bar(full_bar(s), (ks / kSA) & 1, abortp, status, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                // packed rows, 32-byte swizzle: the 16-byte halves of rows with bit 2 set are swapped
                const int sw = (r >> 2) & 1;
                uint32_t regs[32];
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    // explicit shared-memory loads (a generic load waits on the long scoreboard)
                    const uint32_t rowp = sA + (uint32_t)(s * NA + a) * kPackedTile + (uint32_t)r * 32u;
                    const uint4 lo = lds_v4(rowp + 16u * sw);
                    const uint4 hi = lds_v4(rowp + 16u * (sw ^ 1));
                    const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    if (a == 0) {
                        ok = wait_bar(aempty_bar(sa), ((ks / kAStages) & 1) ^ 1, abortp, status, lim);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                    }
#pragma unroll
                    for (int g = 0; g < 8; ++g) unpack_word<GATED>(words[g], &regs[4 * g]);
                    tmem_st32(a_ring + sa * kAStageCols + a * (BK / 2) + lane_off, regs);
                }
                if (!ok) break;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(afull_bar(sa));
                    mbar_arrive(empty_bar(s));
                }
            }
            if (!ok) break;
            // epilogue of this tile
            ok = wait_bar(accfull_bar, tc & 1, abortp, status, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int nmma = (tl.n + 15) & ~15;
            const float s0 = __ldg(tl.sc0 + r);
            const float s1 = GATED ? __ldg(tl.sc1 + r) : 0.0f;
            for (int c0 = 16 * set; c0 < nmma; c0 += 16 * kConvSets) {
                uint32_t v0[16], v1[16], v2[16];
                tmem_ld16(acc0 + c0 + lane_off, v0);
                if (GATED || NI > 1) tmem_ld16(acc1 + c0 + lane_off, v1);
                if (!GATED && NI > 2) tmem_ld16(acc2 + c0 + lane_off, v2);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c0 + i;
                    if (n < tl.n) {
                        if (GATED) {
                            const float xs24 = 24.0f * __ldg(args.xsum_slot + tl.slot0 + n);
                            const float g = s0 * fmaf(16.0f, __uint_as_float(v0[i]), -xs24);
                            const float u = s1 * fmaf(16.0f, __uint_as_float(v1[i]), -xs24);
                            const float hv = g / (1.0f + expf(-g)) * u;
                            const __half hh = __float2half_rn(hv);
                            if (!isfinite(__half2float(hh)) && isfinite(hv)) latch_status(status, MOE_ERR_RANGE);
                            static_cast<uint16_t*>(args.out)[(size_t)(tl.slot0 + n) * args.ld_out + kperm_pos(tl.m0 + r)] =
                                __half_as_ushort(hh);
                        } else {
                            float acc = __uint_as_float(v0[i]);
                            if (NI > 1) acc += __uint_as_float(v1[i]);
                            if (NI > 2) acc += __uint_as_float(v2[i]);
                            static_cast<float*>(args.out)[(size_t)(tl.slot0 + n) * args.ld_out + tl.m0 + r] = s0 * acc;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty_bar);
        }
        if (lane == 0) consumed_sh[warp - 2] = ks;
    }

    __syncthreads();
    // drain TMA copies that were issued but not consumed (only after an abort)
    if (warp == 0 && lane == 0) {
        int consumed = consumed_sh[0];
        for (int i = 1; i < kConvWarps; ++i) consumed = min(consumed, consumed_sh[i]);
        for (int k2 = consumed; k2 < issued_sh; ++k2) wait_bar_drain(full_bar(k2 % kSA), (k2 / kSA) & 1, lim);
        for (int k2 = b_consumed_sh; k2 < b_issued_sh; ++k2)
            wait_bar_drain(bfull_bar(k2 % kBStages), (k2 / kBStages) & 1, lim);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------------------
// gather: xg[slot] = x[token of slot] with K permuted within groups of 8 as [0,4,1,5,2,6,3,7]
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
gather_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, const int32_t* __restrict__ off,
              const double* __restrict__ xsum, int T, int k, int S, int E, int d, uint16_t* __restrict__ xg,
              float* __restrict__ xsum_slot) {
    const int per_row = d / 8;
    const size_t total = (size_t)T * (k + S) * per_row;
    const int n_routed = off[E];          // routed slots in use (adaptive top-p may leave fewer than T k)
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int slot = (int)(i / per_row), c = (int)(i % per_row);
        if (slot < T * k && slot >= n_routed) continue;
        const int t = slot < T * k ? perm[slot] / k : slot - T * k;
        const uint4 v = ld_ro16(x + (size_t)t * d + 8 * c);
        uint4 o;
        o.x = __byte_perm(v.x, v.z, 0x5410);
        o.y = __byte_perm(v.x, v.z, 0x7632);
        o.z = __byte_perm(v.y, v.w, 0x5410);
        o.w = __byte_perm(v.y, v.w, 0x7632);
        reinterpret_cast<uint4*>(xg + (size_t)slot * d)[c] = o;
        if (c == 0) xsum_slot[slot] = (float)xsum[t];
    }
}

// ---------------------------------------------------------------------------------------
// schedule: groups of at most 128 tokens per unique expert (routed first, then shared)
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
schedule_kernel(const int32_t* __restrict__ cnt, const int32_t* __restrict__ off, const int32_t* __restrict__ ulist,
                const int32_t* __restrict__ n_unique_p, int T, int k, int S, Group* __restrict__ groups,
                int* __restrict__ n_groups) {
    __shared__ int scan[1024];
    const int nu = *n_unique_p;
    // each thread owns experts u = 2*tid and 2*tid+1 of the unique list
    int c[2] = {0, 0};
    for (int j = 0; j < 2; ++j) {
        const int u = 2 * threadIdx.x + j;
        if (u < nu) c[j] = (cnt[ulist[u]] + BN - 1) / BN;
    }
    const int mine = c[0] + c[1];
    scan[threadIdx.x] = mine;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int add = threadIdx.x >= o ? scan[threadIdx.x - o] : 0;
        __syncthreads();
        scan[threadIdx.x] += add;
        __syncthreads();
    }
    int g = scan[threadIdx.x] - mine;
    const int nr = scan[1023];
    for (int j = 0; j < 2; ++j) {
        const int u = 2 * threadIdx.x + j;
        if (u >= nu) break;
        const int e = ulist[u], n = cnt[e], o = off[e];
        for (int b = 0; b * BN < n; ++b, ++g) groups[g] = Group{e, o + b * BN, min(BN, n - b * BN), 0};
    }
    if (S) {
        const int ns = (T + BN - 1) / BN;
        for (int b = threadIdx.x; b < ns; b += blockDim.x)
            groups[nr + b] = Group{-1, T * k + b * BN, min(BN, T - b * BN), 0};
        if (threadIdx.x == 0) { n_groups[0] = nr; n_groups[1] = ns; }
    } else if (threadIdx.x == 0) {
        n_groups[0] = nr;
        n_groups[1] = 0;
    }
}

size_t gemm_smem_bytes(bool gated) {
    (void)gated;
    return 1024 + (size_t)kBStages * kBTile + kASmBytes;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D row-major tensor map: inner dimension `cols` elements, `rows` rows, box box_cols x box_rows.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

// Tensor maps of one layer (weights and workspace never move, so they are built once).
struct PrefillPlan {
    CUtensorMap a1, a1_sh, a2, a2_sh;
    CUtensorMap b1[4], b2[4];             // B boxes of 16, 32, 64 and 128 rows
    bool ok = false;
};

bool prefill_supported(const LayerDims& L) {
    return L.wkind == MOE_W_INT4_ROWSCALE && L.d % BM == 0 && L.f % BM == 0 && (!L.S || L.f_shared % BM == 0) &&
           L.E * 2 * L.f <= (1 << 30);
}

PrefillPlan* prefill_plan_create(const LayerDims& L, const moe_weights& W, const Workspace& ws, int max_tokens) {
    if (!prefill_supported(L)) return nullptr;
    PrefillPlan* p = new PrefillPlan();
    const uint64_t slots = (uint64_t)max_tokens * (L.k + L.S);
    const int fmax = L.S && L.f_shared > L.f ? L.f_shared : L.f;
    bool ok = true;
    ok &= make_map(&p->a1, W.gate_up, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.d / 2, (uint64_t)L.E * 2 * L.f, BK / 2, BM,
                   CU_TENSOR_MAP_SWIZZLE_32B);
    ok &= make_map(&p->a2, W.down, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.f / 2, (uint64_t)L.E * L.d, BK / 2, BM,
                   CU_TENSOR_MAP_SWIZZLE_32B);
    if (L.S) {
        ok &= make_map(&p->a1_sh, W.shared_gate_up, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.d / 2, 2 * (uint64_t)L.f_shared,
                       BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_32B);
        ok &= make_map(&p->a2_sh, W.shared_down, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.f_shared / 2, (uint64_t)L.d,
                       BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_32B);
    } else {
        p->a1_sh = p->a1;
        p->a2_sh = p->a2;
    }
    for (int i = 0; i < 4; ++i) {
        const uint32_t rows = 16u << i;
        ok &= make_map(&p->b1[i], ws.xg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L.d, slots, BK, rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
        ok &= make_map(&p->b2[i], ws.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, fmax, slots, BK, rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    }
    p->ok = ok;
    if (!ok) {
        delete p;
        return nullptr;
    }
    return p;
}

void prefill_plan_destroy(PrefillPlan* p) { delete p; }

cudaError_t prepare_prefill(const LayerDims& L) {
    if (!prefill_supported(L)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemm_smem_bytes(true));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_smem_bytes(false));
    return e;
}

size_t prefill_max_groups(const LayerDims& L, int max_tokens) {
    return (size_t)L.E + ((size_t)max_tokens * L.k + BN - 1) / BN + ((size_t)max_tokens + BN - 1) / BN + 2;
}

cudaError_t launch_prefill_experts(const LayerDims& L, const PrefillPlan* p, const moe_weights& W, const uint16_t* x,
                                   int T, const Workspace& ws, int num_sms, const Launch& ctx) {
    if (T == 0) return cudaSuccess;
    const int fmax = L.S && L.f_shared > L.f ? L.f_shared : L.f;
    Group* groups = reinterpret_cast<Group*>(ws.groups);
    QE_LAUNCH(ctx, MOE_KERNEL_GATHER,
              (schedule_kernel<<<1, 1024, 0, ctx.s>>>(ws.cnt, ws.off, ws.ulist, ws.n_unique, T, L.k, L.S, groups,
                                                      ws.n_groups)));
    const size_t work = (size_t)T * (L.k + L.S) * (L.d / 8);
    const unsigned gg = (unsigned)std::min<size_t>((work + 255) / 256, (size_t)num_sms * 16);
    QE_LAUNCH(ctx, MOE_KERNEL_GATHER,
              (gather_kernel<<<gg, 256, 0, ctx.s>>>(x, ws.perm, ws.off, ws.xsum, T, L.k, L.S, L.E, L.d, ws.xg,
                                                    ws.xsum_slot)));
    GemmArgs a1{groups, ws.n_groups, W.gate_up_scale, W.shared_gate_up_scale, 2 * L.f, L.f, L.S ? L.f_shared : L.f,
                L.f / BM, L.S ? L.f_shared / BM : 1, L.d, L.d, fmax, ws.h, ws.status, ws.xsum_slot, L.wait_ns,
                L.test_skip_b};
    QE_LAUNCH(ctx, MOE_KERNEL_GEMM_GATEUP,
              (gemm_kernel<true><<<num_sms, kGemmThreads, gemm_smem_bytes(true), ctx.s>>>(
                  p->a1, p->a1_sh, p->b1[0], p->b1[1], p->b1[2], p->b1[3], a1)));
    GemmArgs a2{groups, ws.n_groups, W.down_scale, W.shared_down_scale, L.d, L.f, L.S ? L.f_shared : L.f,
                L.d / BM, L.d / BM, L.f, L.S ? L.f_shared : L.f, L.d, ws.Y, ws.status, nullptr, L.wait_ns,
                L.test_skip_b};
    QE_LAUNCH(ctx, MOE_KERNEL_GEMM_DOWN,
              (gemm_kernel<false><<<num_sms, kGemmThreads, gemm_smem_bytes(false), ctx.s>>>(
                  p->a2, p->a2_sh, p->b2[0], p->b2[1], p->b2[2], p->b2[3], a2)));
    return cudaSuccess;
}

}  // namespace qe
