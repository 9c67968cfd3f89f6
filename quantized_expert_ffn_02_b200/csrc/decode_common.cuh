// decode_common.cuh -- pieces shared by the single-token decode kernels: mbarrier waits with a
// time limit, TMA bulk copies into shared memory, and the nibble dequantisation dot products.
#pragma once

#include "internal.cuh"

namespace qe {
namespace dec {

constexpr uint32_t kNib = 0x000F000Fu;
// With lop_sel_xor(word, kNib, magic), nibble n of signed code s (n = s & 15, so n ^ 8 = s + 8)
// lands in the low mantissa bits, where one unit is 1:
constexpr uint32_t kBf16Magic = 0x43084308u;   // bf16 136 in each half: the pair reads 128 + (n ^ 8) = 136 + s
constexpr uint32_t kF16Magic = 0x64086408u;    // fp16 1032 in each half: 1024 + (n ^ 8) = 1032 + s; minus 1032 is s
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(n));
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
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
// The same test, but the thread may sleep in the instruction (up to about 1 ms) until the phase
// completes, instead of spinning and taking issue slots from the warps that compute.
__device__ __forceinline__ bool bar_try_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait (every lane of the warp calls it; the result is made uniform by the caller).
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    if (bar_try(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    while (!bar_try_sleep(bar, parity))
        if (now_ns() - t0 > kWaitLimitNs) return false;
    return true;
}
// Bulk copy global -> shared, completion counted on `bar`.  16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ uint4 lds16(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts16(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// 8 bf16 of columns 8m..8m+7 -> four registers holding (col i, col i+4), i = 0..3
__device__ __forceinline__ void pair_cols(const uint4 v, uint32_t* p) {
    p[0] = __byte_perm(v.x, v.z, 0x5410);
    p[1] = __byte_perm(v.x, v.z, 0x7632);
    p[2] = __byte_perm(v.y, v.w, 0x5410);
    p[3] = __byte_perm(v.y, v.w, 0x7632);
}

// acc += sum over the 8 codes of word w of (136 + s) * x (x pairs matching the nibble pairs)
__device__ __forceinline__ float dot_word_bf16(uint32_t w, const uint32_t* xp, float acc) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t p = lop_sel_xor(w >> (4 * i), kNib, kBf16Magic);
        unsigned short wl, wh, xl, xh;
        halves(p, wl, wh);
        halves(xp[i], xl, xh);
        acc = fma_bf16(wl, xl, acc);
        acc = fma_bf16(wh, xh, acc);
    }
    return acc;
}

// acc += sum over the 8 codes of word w of s * h (h pairs matching the nibble pairs)
__device__ __forceinline__ float dot_word_f16(uint32_t w, const uint32_t* hp, float acc) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t p = hsub2_u32(lop_sel_xor(w >> (4 * i), kNib, kF16Magic), kF16Magic);
        unsigned short wl, wh, hl, hh;
        halves(p, wl, wh);
        halves(hp[i], hl, hh);
        acc = fma_f16(wl, hl, acc);
        acc = fma_f16(wh, hh, acc);
    }
    return acc;
}

// acc += sum over the 8 codes of word w of (3/2 + s/16) * h.  The nibble goes to the top four
// mantissa bits of an fp16 1.0 (mask 0x03C0 per half), so the pair reads 1 + (n ^ 8) / 16 =
// 3/2 + s/16 exactly, one shift and one LOP3 per pair and no subtraction.  The caller recovers
// sum s h = 16 acc - 24 sum h; the offset is small next to the codes, so the cancellation costs
// only a few units of fp32 rounding.
constexpr uint32_t kF16TopMask = 0x03C003C0u;
constexpr uint32_t kF16TopMagic = 0x3E003E00u;   // fp16 1.5 in each half: bit 9 flips the nibble's sign
__device__ __forceinline__ float dot_word_f16top(uint32_t w, const uint32_t* hp, float acc) {
    const uint32_t src[4] = {w << 6, w << 2, w >> 2, w >> 6};   // nibble pair i -> bits 6..9, 22..25
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t p = lop_sel_xor(src[i], kF16TopMask, kF16TopMagic);
        unsigned short wl, wh, hl, hh;
        halves(p, wl, wh);
        halves(hp[i], hl, hh);
        acc = fma_f16(wl, hl, acc);
        acc = fma_f16(wh, hh, acc);
    }
    return acc;
}

// Launch that may start while the previous kernel on the stream is still running (when
// `programmatic`); the kernel itself waits (griddepcontrol.wait) before reading that kernel's
// results.  Without the attribute the wait returns at once.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(bool programmatic, Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace dec
}  // namespace qe
