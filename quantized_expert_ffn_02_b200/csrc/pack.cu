// pack.cu -- K1: fp32 -> packed int4 (and the int8 / packed int2 tiers) with one fp32 scale per row.
//
// The container of the colibri README ("What's implemented": int8 / packed int4 / packed
// int2, per-row scales, dequant-on-use; packing validated bit-identical to the int8
// container): per row, scale = fp32(max|w| / 7) by IEEE division, code = round-half-even of
// the fp32 quotient w / scale, clamped to [-8, 7]; two 4-bit two's-complement codes per
// byte, the even column in the low nibble.  Division and rounding are exactly specified
// operations, so these bytes equal any correct implementation's bytes.
#include "internal.cuh"

namespace qe {
namespace {

constexpr int kPackThreads = 256;

__device__ __forceinline__ uint32_t code4(float v, float s) {
    float q = 0.0f;
    if (s != 0.0f && isfinite(v)) q = rintf(__fdiv_rn(v, s));
    q = fminf(fmaxf(q, -8.0f), 7.0f);
    return (uint32_t)((int)q) & 0xFu;
}

__device__ __forceinline__ float block_max(float v, float* red) {
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
    const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float m = 0.0f;
    for (int i = 0; i < (int)blockDim.x / kWarp; ++i) m = fmaxf(m, red[i]);
    return m;
}

// One block per row (grid-stride).  `vec8` selects the path where a thread packs 8 columns
// (two 16-byte loads, one 4-byte store); it needs cols % 8 == 0 and 16/4-byte alignment.
__global__ void __launch_bounds__(kPackThreads)
pack_int4_kernel(const float* __restrict__ w, int64_t rows, int64_t cols, uint8_t* __restrict__ packed,
                 float* __restrict__ scales, int* status, int vec8) {
    __shared__ float red[kPackThreads / kWarp];
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const float* row = w + r * cols;
        float m = 0.0f;
        int bad = 0;
        if (vec8) {
            const float4* row4 = reinterpret_cast<const float4*>(row);
            for (int64_t c = threadIdx.x; c < cols / 4; c += blockDim.x) {
                float4 v = row4[c];
                bad |= !isfinite(v.x) | !isfinite(v.y) | !isfinite(v.z) | !isfinite(v.w);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            }
        } else {
            for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
                float v = row[c];
                bad |= !isfinite(v);
                m = fmaxf(m, fabsf(v));
            }
        }
        const int bad_any = __syncthreads_or(bad);
        m = block_max(m, red);                // contains __syncthreads
        const float s = __fdiv_rn(m, 7.0f);
        if (threadIdx.x == 0) {
            scales[r] = s;
            if (bad_any) latch_status(status, MOE_ERR_RANGE);
        }
        uint8_t* prow = packed + r * (cols / 2);
        if (vec8) {
            const float4* row4 = reinterpret_cast<const float4*>(row);
            uint32_t* prow4 = reinterpret_cast<uint32_t*>(prow);
            for (int64_t c = threadIdx.x; c < cols / 8; c += blockDim.x) {
                float4 a = row4[2 * c], b = row4[2 * c + 1];
                uint32_t word = code4(a.x, s) | (code4(a.y, s) << 4) | (code4(a.z, s) << 8) |
                                (code4(a.w, s) << 12) | (code4(b.x, s) << 16) | (code4(b.y, s) << 20) |
                                (code4(b.z, s) << 24) | (code4(b.w, s) << 28);
                prow4[c] = word;
            }
        } else {
            for (int64_t j = threadIdx.x; j < cols / 2; j += blockDim.x)
                prow[j] = (uint8_t)(code4(row[2 * j], s) | (code4(row[2 * j + 1], s) << 4));
        }
        __syncthreads();
    }
}

// The b-bit tier (b = 8 or 2) of the same rule: scale = fp32(max|w| / qmax), qmax = 2^(b-1) - 1,
// code = round-half-even(fp32(w / scale)) clamped to [-qmax - 1, qmax].  b = 8: one code per byte
// (the int8 container); b = 2: four codes per byte, column 4j + i in bits 2i .. 2i+1 of byte j.
// One block per row; a thread writes one 32-bit word (4 or 16 columns) when cols allows it.
template <int BITS>
__global__ void __launch_bounds__(kPackThreads)
pack_tier_kernel(const float* __restrict__ w, int64_t rows, int64_t cols, uint8_t* __restrict__ packed,
                 float* __restrict__ scales, int* status, int vecw) {
    constexpr int PER_BYTE = 8 / BITS;
    constexpr float kQmax = (float)((1 << (BITS - 1)) - 1);
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    __shared__ float red[kPackThreads / kWarp];
    auto code = [](float v, float s) -> uint32_t {
        float q = 0.0f;
        if (s != 0.0f && isfinite(v)) q = rintf(__fdiv_rn(v, s));
        q = fminf(fmaxf(q, -kQmax - 1.0f), kQmax);
        return (uint32_t)((int)q) & kMask;
    };
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const float* row = w + r * cols;
        float m = 0.0f;
        int bad = 0;
        for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
            const float v = row[c];
            bad |= !isfinite(v);
            m = fmaxf(m, fabsf(v));
        }
        const int bad_any = __syncthreads_or(bad);
        m = block_max(m, red);                // contains __syncthreads
        const float s = __fdiv_rn(m, kQmax);
        if (threadIdx.x == 0) {
            scales[r] = s;
            if (bad_any) latch_status(status, MOE_ERR_RANGE);
        }
        uint8_t* prow = packed + r * (cols / PER_BYTE);
        if (vecw) {
            constexpr int CPW = 4 * PER_BYTE;   // columns per 32-bit word
            uint32_t* prow4 = reinterpret_cast<uint32_t*>(prow);
            for (int64_t c = threadIdx.x; c < cols / CPW; c += blockDim.x) {
                uint32_t word = 0;
#pragma unroll
                for (int i = 0; i < CPW; ++i) word |= code(row[CPW * c + i], s) << (BITS * i);
                prow4[c] = word;
            }
        } else {
            for (int64_t j = threadIdx.x; j < cols / PER_BYTE; j += blockDim.x) {
                uint32_t b = 0;
#pragma unroll
                for (int i = 0; i < PER_BYTE; ++i) b |= code(row[PER_BYTE * j + i], s) << (BITS * i);
                prow[j] = (uint8_t)b;
            }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_pack_tier(int bits, const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                             int* status, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int per_word = bits == 8 ? 4 : 16;
    const int vecw = (cols % per_word == 0) && (((uintptr_t)packed & 3) == 0);
    int64_t grid = rows < 148 * 16 ? rows : 148 * 16;
    if (bits == 8)
        pack_tier_kernel<8><<<(unsigned)grid, kPackThreads, 0, s>>>(w, rows, cols, packed, scales, status, vecw);
    else
        pack_tier_kernel<2><<<(unsigned)grid, kPackThreads, 0, s>>>(w, rows, cols, packed, scales, status, vecw);
    return cudaGetLastError();
}

cudaError_t launch_pack_int4(const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                             int* status, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int vec8 = (cols % 8 == 0) && (((uintptr_t)w & 15) == 0) && (((uintptr_t)packed & 3) == 0);
    int64_t grid = rows < 148 * 16 ? rows : 148 * 16;
    pack_int4_kernel<<<(unsigned)grid, kPackThreads, 0, s>>>(w, rows, cols, packed, scales, status, vec8);
    return cudaGetLastError();
}

}  // namespace qe
