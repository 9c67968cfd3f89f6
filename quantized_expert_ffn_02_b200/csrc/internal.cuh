// internal.cuh -- device helpers and the launch interface shared by the kernels of libmoe.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace qe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------------------
// Status word: the first error a kernel meets is latched (later ones are dropped).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void latch_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------------------
// 16-bit lanes of a 32-bit register and mixed-precision FMA (f32 += bf16*bf16 / f16*f16).
// The product of two 16-bit floats is exact in the fused operation; only the sum rounds.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void halves(uint32_t v, unsigned short& lo, unsigned short& hi) {
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(v));
}
__device__ __forceinline__ float fma_bf16(unsigned short a, unsigned short b, float c) {
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_f16(unsigned short a, unsigned short b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}
// (a & b) | (~b & ... ) -- the 3-input function  b ? (a ^ c) : c, one LOP3.
// With b = 0x000F000F it keeps the low nibble of each 16-bit half, flips the bits where c
// has a 1 inside that nibble, and copies c elsewhere.
__device__ __forceinline__ uint32_t lop_sel_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Streaming 16-byte load (read once: do not keep in L1).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
// Coherent 16-byte load through L2 only.  Required for data written by a kernel whose lifetime
// overlaps the reader's (programmatic dependent launch): the .nc path may serve stale lines.
__device__ __forceinline__ uint4 ld_cg16(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p) : "memory");
    return v;
}
// Read-only 16-byte load that may stay in L1 (activations reused by many warps).  Only for data
// that no kernel running at the same time can write.
__device__ __forceinline__ uint4 ld_ro16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float bf16_bits_to_f32(unsigned short b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

}  // namespace qe

// ---------------------------------------------------------------------------------------
// Launch interface (host functions defined next to their kernels).
// ---------------------------------------------------------------------------------------
namespace qe {

struct Workspace {
    double* logits;        // [maxT][E]
    int32_t* idx;          // [maxT][k]   rank order
    float* wts;            // [maxT][k]
    int32_t* asc;          // [maxT][k]   ranks of a token's experts in ascending expert order
    double* xsum;          // [maxT]      sum of x over the hidden dimension
    int32_t* cnt;          // [E]
    int32_t* off;          // [E + 1]
    int32_t* perm;         // [maxT * k]  routed slot -> entry (t * k + rank)
    int32_t* slot_of;      // [maxT * k]  entry -> routed slot
    int32_t* ulist;        // [E]         unique chosen experts, ascending
    int32_t* n_unique;     // [1]
    uint16_t* h;           // [slots][fmax] fp16 bits: SwiGLU activations
    float* Y;              // [slots][d]   per-slot expert outputs (before the gate weight)
    int32_t* status;       // [1]
    // grouped-GEMM (prefill) path
    uint16_t* xg;          // [slots][d] bf16: x gathered per slot, K order permuted in groups of 8
    int32_t* groups;       // [max_groups][4]: (expert or -1, first slot, tokens, unused)
    int32_t* n_groups;     // [2]: routed groups, shared groups
    float* xsum_slot;      // [slots]: sum of x of each slot's token (gate/up GEMM epilogue)
    uint32_t* counter;     // [1]: blocks done in the fused small-batch router (reset to 0 by the last)
    // single-launch decode path
    // the routed experts' weights, one pointer each: [0, E) gate/up rows, [E, 2E) gate/up scales,
    // [2E, 3E) down rows, [3E, 4E) down scales.  Filled from the contiguous [E] arrays at layer
    // creation; moe_layer_set_expert re-points one expert (a non-contiguous expert slab).
    const void** etab;
    double* rpart;         // [2][E][d / 1024]: pieces of the router logits of one or two tokens
    double* rsplit;        // partial logits and sums of x of the K-sliced router GEMM
    double* keys;          // [T][E] selection keys (small-batch router)
    double* rsmall;        // small-batch router: [slices][T][E] partial logits, [slices][T] partial x sums
    unsigned int* rsmall_cnt;   // small-batch router: finished blocks per expert group
    size_t rsplit_n;       // its length in doubles (0: none)
    unsigned long long* gbar;  // [1]: grid-barrier arrivals (only grows)
    unsigned long long* trace; // [kTraceCtas][kTraceStamps]: phase timestamps of that path
};
constexpr int kTraceCtas = 1024;
constexpr int kTraceStamps = 16;

// Router variants (colibri README: the DeepSeek-V3 router's noaux_tc, and the --topp adaptive
// expert top-p knob): group-limited selection when n_group > 1 -- the E experts form n_group
// contiguous groups, a group's score is the sum of its two largest keys, and only the topk_group
// best groups (equal scores: the lower group first) stay selectable -- and, for top_p in (0, 1),
// the shortest rank-order prefix whose weights reach top_p of the k weights' total, rescaled to
// that total, the rest dropped (index -1, weight 0).  The defaults are the plain router.
struct RouterOpts {
    int n_group = 1, topk_group = 1;
    double top_p = 0.0;
    bool active() const { return n_group > 1 || (top_p > 0.0 && top_p < 1.0); }
};

// Routed expert e's weights through the layer's pointer table ([4][E]; no kernel writes it while
// another reads it, so it goes through the read-only cache).
__device__ __forceinline__ const uint8_t* ex_gate_up(const void* const* t, int E, int e) {
    return reinterpret_cast<const uint8_t*>(__ldg(reinterpret_cast<const unsigned long long*>(t) + e));
}
__device__ __forceinline__ const float* ex_gu_scale(const void* const* t, int E, int e) {
    return reinterpret_cast<const float*>(__ldg(reinterpret_cast<const unsigned long long*>(t) + E + e));
}
__device__ __forceinline__ const uint8_t* ex_down(const void* const* t, int E, int e) {
    return reinterpret_cast<const uint8_t*>(__ldg(reinterpret_cast<const unsigned long long*>(t) + 2 * E + e));
}
__device__ __forceinline__ const float* ex_dn_scale(const void* const* t, int E, int e) {
    return reinterpret_cast<const float*>(__ldg(reinterpret_cast<const unsigned long long*>(t) + 3 * E + e));
}

struct LayerDims {
    int d, f, E, k, S, f_shared, router, wkind, out_bf16;
    float scaling;
    int pdl = 1;           // chain dependent kernels with programmatic dependent launch
    uint64_t wait_ns = 2000000000ull;   // limit of the grouped-GEMM kernels' bounded waits
    int test_skip_b = 0;   // test hook: the grouped GEMM's B producer issues no copies
    int phase_trace = 0;   // the single launch records its phase times
    RouterOpts ropts;      // router variants (off by default)
};

// Optional per-kernel event timing (defined in layer.cu).  `prof` may be null.
struct Profiler;
void prof_mark(Profiler* prof, int kernel, bool begin, cudaStream_t s);

// What every launch function needs: the stream, the launch counter, the profiler.
struct Launch {
    cudaStream_t s;
    int* launches;
    Profiler* prof;
};

// Per-device, per-layer set-up (shared-memory opt-ins); called by moe_layer_create.
cudaError_t prepare_router(const LayerDims& L);
cudaError_t prepare_bucket(const LayerDims& L);
cudaError_t prepare_decode(const LayerDims& L);

cudaError_t launch_pack_int4(const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                             int* status, cudaStream_t s);
// bits = 8 (int8 container) or 2 (packed int2)
cudaError_t launch_pack_tier(int bits, const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                             int* status, cudaStream_t s);
// part (nullable, part_doubles long): room for the K-sliced router GEMM's partial logits and sums
// of x; router_split_doubles gives the size that lets every batch up to max_tokens use it.
cudaError_t launch_router(const LayerDims& L, const float* router_w, const float* router_bias,
                          const uint16_t* x, int T, double* logits, double* xsum, int32_t* idx, float* wts,
                          int32_t* asc, const Launch& ctx, double* part, size_t part_doubles);
size_t router_split_doubles(int E, int max_tokens);
cudaError_t launch_bucket(const LayerDims& L, int T, const Workspace& ws, const Launch& ctx);
// Small batches (T >= 2), int4 experts with d, f (and the shared f) multiples of 1024: gate/up and
// down as 16-row x 8-token tensor-core products (decode_mma.cu).
bool decode_mma_ok(const LayerDims& L, int T);
cudaError_t prepare_decode_mma();
cudaError_t launch_decode_mma(const LayerDims& L, const moe_weights& W, const uint16_t* x, int T, const Workspace& ws,
                              int num_sms, const Launch& ctx);
// Small batches: logits, top-k, gate weights and bucket tables in one launch.
constexpr int kRouteSmallMaxT = 32;
bool route_small_ok(const LayerDims& L, int num_sms);
size_t route_small_part_doubles(int E, int max_tokens);
size_t route_small_groups(int E);
cudaError_t launch_route_small(const LayerDims& L, const float* router_w, const float* router_bias, const uint16_t* x,
                               int T, const Workspace& ws, int num_sms, const Launch& ctx);
// One token, int4 experts: gate/up and down+combine kernels (decode1.cu).
bool decode_t1_supported(const LayerDims& L);
cudaError_t launch_decode_t1(const LayerDims& L, const moe_weights& W, const uint16_t* x, const Workspace& ws,
                             void* out, int num_sms, const Launch& ctx);
// One or two tokens (nt), int4 experts (bf16 too for one token), the whole layer in one
// cooperative launch (decode_fused.cu).
bool decode_fused_shape_ok(const LayerDims& L, int nt);
cudaError_t prepare_decode_fused(const LayerDims& L, int num_sms, bool* usable, int nt);
cudaError_t launch_decode_fused(const LayerDims& L, const moe_weights& W, const uint16_t* x, const Workspace& ws,
                                void* out, int num_sms, const Launch& ctx, int nt);
cudaError_t launch_decode_experts(const LayerDims& L, const moe_weights& W, const uint16_t* x, int T,
                                  const Workspace& ws, int num_sms, const Launch& ctx);
cudaError_t launch_combine(const LayerDims& L, int T, const Workspace& ws, void* out, const Launch& ctx);

// Grouped-GEMM path (prefill.cu).  A plan holds the layer's TMA tensor maps.
struct PrefillPlan;
bool prefill_supported(const LayerDims& L);
size_t prefill_max_groups(const LayerDims& L, int max_tokens);
cudaError_t prepare_prefill(const LayerDims& L);
PrefillPlan* prefill_plan_create(const LayerDims& L, const moe_weights& W, const Workspace& ws, int max_tokens);
void prefill_plan_destroy(PrefillPlan* p);
cudaError_t launch_prefill_experts(const LayerDims& L, const PrefillPlan* p, const moe_weights& W, const uint16_t* x,
                                   int T, const Workspace& ws, int num_sms, const Launch& ctx);

// Launch bookkeeping shared by the launch functions: profiler marks and the launch count.
#define QE_LAUNCH(ctx, kernel_id, ...)                       \
    do {                                                     \
        prof_mark((ctx).prof, (kernel_id), true, (ctx).s);   \
        __VA_ARGS__;                                         \
        cudaError_t qe_err_ = cudaGetLastError();            \
        prof_mark((ctx).prof, (kernel_id), false, (ctx).s);  \
        if (qe_err_ != cudaSuccess) return qe_err_;          \
        ++*(ctx).launches;                                   \
    } while (0)

}  // namespace qe
