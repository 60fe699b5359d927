// FP8 (e4m3) latent cache: the format and its encode / decode helpers.
//
// "MLA架构：低秩注意力机制优化LLM显存与计算效率" section 4.2 (item 3, "量化的影响")
// notes that quantising the cache shrinks it further; the page fixes no
// format, so this library defines one:
//   - each latent value is an OCP E4M3 code (bias 7, subnormals, max 448,
//     S.1111.111 = NaN) of c / s_t, rounded to nearest even and saturated;
//   - s_t = 2^e_t, one per token, e_t the smallest integer with
//     max|c_t| <= 448 * 2^e_t, clamped to [-15, 7]: dividing by it is exact,
//     and every code * s_t is exactly an IEEE half, so the attention kernel
//     dequantises into f16 operands without rounding;
//   - the RoPE key k_pe is stored as f16 (rounded to nearest even);
//   - a cache block of block_size tokens is block_size rows of
//     d_c + 2 d_r bytes (codes, then the f16 key), followed by the block's
//     block_size fp32 scales. DeepSeek-V3: 64 * 640 + 256 = 41216 bytes per
//     block, 644 bytes per token instead of 1152.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace mla {
namespace fp8 {

constexpr float kE4M3Max = 448.f;
constexpr int kExpMin = -15, kExpMax = 7;

__host__ __device__ constexpr int64_t row_bytes(int dc, int dr) { return dc + 2 * dr; }
__host__ __device__ constexpr int64_t block_bytes(int dc, int dr, int bs) { return bs * (row_bytes(dc, dr) + 4); }

// 2^e as a float (e in the normal exponent range).
__device__ __forceinline__ float pow2(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }

// The smallest e in [kExpMin, kExpMax] with amax <= 448 * 2^e (amax >= 0). The
// start, floor(log2 amax) - 9, is never enough (448 * 2^(p - 9) < 2^p <= amax),
// so at most two steps follow; 448 * 2^e is exact in fp32.
__device__ __forceinline__ int scale_exp(float amax) {
    const int p = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
    int e = min(max(kExpMin, p - 9), kExpMax);
    while (e < kExpMax && amax > kE4M3Max * pow2(e)) ++e;
    return e;
}

// Two floats to e4m3 codes (nearest even, saturated to +-448): lo in bits 0-7.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two e4m3 codes (bits 0-7 and 8-15) to their exact f16 values (lo half first).
__device__ __forceinline__ uint32_t f16x2_of_e4m3x2(uint32_t two_codes) {
    uint32_t r;
    const uint16_t v = static_cast<uint16_t>(two_codes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Four codes (one word, byte i = code i) times the f16x2 scale s2: the four
// dequantised values as f16, codes 0-1 in .x and 2-3 in .y. Exact: the scale is
// a power of two and every product is a half (see the format above).
__device__ __forceinline__ uint2 dequant4(uint32_t codes, uint32_t s2) {
    return make_uint2(hmul2(f16x2_of_e4m3x2(codes & 0xFFFFu), s2), hmul2(f16x2_of_e4m3x2(codes >> 16), s2));
}

__device__ __forceinline__ uint16_t f16_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }

// The f16x2 word (s, s) of a scale 2^e, e in [kExpMin, kExpMax].
__device__ __forceinline__ uint32_t scale_f16x2(float s) {
    const uint32_t h = f16_bits(s);
    return h | (h << 16);
}

// Byte offsets of pool row `row` (= block * block_size + slot) in the FP8 layout.
struct Layout {
    int64_t row_b, block_b;
    int32_t bs;
    __device__ int64_t row_off(int64_t row) const { return (row / bs) * block_b + (row % bs) * row_b; }
    __device__ int64_t scale_off(int64_t row) const { return (row / bs) * block_b + bs * row_b + 4 * (row % bs); }
};

// bf16 pool -> FP8 pool, one warp per pool row (both pools hold the same
// num_blocks * block_size rows). dc a multiple of 8, dr even.
// grid ceil(rows / 8); block 256.
__global__ void __launch_bounds__(256) quantize_pool_kernel(const uint16_t* __restrict__ src, int64_t rows, int32_t dc,
                                                           int32_t dr, Layout L, uint8_t* __restrict__ dst) {
    pdl_wait();
    pdl_trigger();
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const uint16_t* s = src + row * (dc + dr);
    float amax = 0.f;
    for (int i = lane; i < dc / 8; i += 32) {
        const uint4 u = *reinterpret_cast<const uint4*>(s + 8 * i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_to_f32(w[k] & 0xFFFFu)), fabsf(bf16_to_f32(w[k] >> 16))));
    }
    amax = warp_max(amax);
    const int e = scale_exp(amax);
    const float inv = pow2(-e);  // exact division by the scale
    uint8_t* d = dst + L.row_off(row);
    for (int i = lane; i < dc / 8; i += 32) {
        const uint4 u = *reinterpret_cast<const uint4*>(s + 8 * i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t q[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint32_t a = e4m3x2(bf16_to_f32(w[2 * k] & 0xFFFFu) * inv, bf16_to_f32(w[2 * k] >> 16) * inv);
            const uint32_t b = e4m3x2(bf16_to_f32(w[2 * k + 1] & 0xFFFFu) * inv, bf16_to_f32(w[2 * k + 1] >> 16) * inv);
            q[k] = a | (b << 16);
        }
        *reinterpret_cast<uint2*>(d + 8 * i) = make_uint2(q[0], q[1]);
    }
    uint32_t* pe = reinterpret_cast<uint32_t*>(d + dc);
    for (int i = lane; i < dr / 2; i += 32) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(s + dc + 2 * i);
        pe[i] = static_cast<uint32_t>(f16_bits(bf16_to_f32(v & 0xFFFFu))) |
                (static_cast<uint32_t>(f16_bits(bf16_to_f32(v >> 16))) << 16);
    }
    if (lane == 0) *reinterpret_cast<float*>(dst + L.scale_off(row)) = pow2(e);
}

}  // namespace fp8
}  // namespace mla
