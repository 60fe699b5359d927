// Log-sum-exp combine of split-KV partials, alone and fused with the
// per-head value up-projection out[g, h] = W_UV[h] o_lat[g, h].
//
// Partial i of (group g, head h) holds o_i (already divided by its own
// softmax denominator) and lse_i = m_i + ln(l_i). The merged result is
//   M = max_i lse_i,  w_i = exp(lse_i - M),  o = sum_i w_i o_i / sum_i w_i,
//   lse = M + ln(sum_i w_i);
// parts with lse = -inf have weight 0, and a group with no finite part
// yields zeros and lse = -inf.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kMaxMergeParts = 64;  // parts merged per pass; more are folded in chunks

// Merge weights of one (g, h); returns sum of weights (0 if none) and writes
// the per-part weights for parts [p0, p0 + n) into w (n <= kMaxMergeParts) relative to M.
__device__ __forceinline__ float merge_max(const float* __restrict__ lse_part, int32_t H, int32_t h,
                                           int32_t p0, int32_t p1) {
    float M = -INFINITY;
    for (int32_t p = p0; p < p1; ++p) M = fmaxf(M, lse_part[static_cast<int64_t>(p) * H + h]);
    return M;
}

// grid (G * H); block 128. o_lat [G, H, dc] fp32, lse_out [G, H] or null.
__global__ void __launch_bounds__(128) combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    const int32_t* __restrict__ part_offsets, int32_t G, int32_t H, int32_t dc,
    float* __restrict__ o_lat, float* __restrict__ lse_out) {
    pdl_wait();
    pdl_trigger();
    const int64_t gh = blockIdx.x;
    const int32_t g = static_cast<int32_t>(gh / H), h = static_cast<int32_t>(gh - static_cast<int64_t>(g) * H);
    const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
    const float M = merge_max(lse_part, H, h, p0, p1);
    float den = 0.f;
    if (M != -INFINITY)
        for (int32_t p = p0; p < p1; ++p) den += __expf(lse_part[static_cast<int64_t>(p) * H + h] - M);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int j = threadIdx.x; j < dc; j += blockDim.x) {
        float acc = 0.f;
        if (den > 0.f)
            for (int32_t p = p0; p < p1; ++p) {
                const float l = lse_part[static_cast<int64_t>(p) * H + h];
                const float w = l == -INFINITY ? 0.f : __expf(l - M);
                acc = fmaf(w, o_part[(static_cast<int64_t>(p) * H + h) * dc + j], acc);
            }
        o_lat[gh * dc + j] = acc * inv;
    }
    if (lse_out && threadIdx.x == 0) lse_out[gh] = den > 0.f ? M + __logf(den) : -INFINITY;
}

constexpr int kUvGroups = 16;   // groups per CTA in the fused combine + up-projection
constexpr int kUvThreads = 256;

// Fused combine + W_UV: grid (H, ceil(G / kUvGroups)), block 256,
// dynamic smem kUvGroups * dc floats. out bf16 [G, H, dv].
__global__ void __launch_bounds__(kUvThreads) combine_uv_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    const int32_t* __restrict__ part_offsets, const uint16_t* __restrict__ w_uv,
    int32_t G, int32_t H, int32_t dc, int32_t dv, uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float ol[];  // [kUvGroups][dc]
    __shared__ float s_w[kUvGroups][kMaxMergeParts];
    __shared__ float s_inv[kUvGroups];
    const int h = blockIdx.x;
    const int g0 = blockIdx.y * kUvGroups;
    const int ng = min(kUvGroups, G - g0);
    // 1) merge partials of each group into ol[gg][:]
    for (int gg = 0; gg < ng; ++gg) {
        const int32_t g = g0 + gg;
        const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
        float* dst = ol + gg * dc;
        for (int j = threadIdx.x; j < dc; j += blockDim.x) dst[j] = 0.f;
        const float M = merge_max(lse_part, H, h, p0, p1);
        float den = 0.f;
        for (int32_t c0 = p0; c0 < p1; c0 += kMaxMergeParts) {
            const int32_t c1 = min(p1, c0 + kMaxMergeParts);
            __syncthreads();
            if (threadIdx.x < c1 - c0) {
                const float l = lse_part[static_cast<int64_t>(c0 + threadIdx.x) * H + h];
                s_w[gg][threadIdx.x] = (M == -INFINITY || l == -INFINITY) ? 0.f : __expf(l - M);
            }
            __syncthreads();
            for (int32_t p = c0; p < c1; ++p) den += s_w[gg][p - c0];
            for (int j = threadIdx.x; j < dc; j += blockDim.x) {
                float acc = dst[j];
                for (int32_t p = c0; p < c1; ++p)
                    acc = fmaf(s_w[gg][p - c0], o_part[(static_cast<int64_t>(p) * H + h) * dc + j], acc);
                dst[j] = acc;
            }
        }
        if (threadIdx.x == 0) s_inv[gg] = den > 0.f ? 1.f / den : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ng * dc; i += blockDim.x) ol[i] *= s_inv[i / dc];
    __syncthreads();
    // 2) out[g, h, i] = sum_j W_UV[h, i, j] * o_lat[g, h, j]; one warp per output row i
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const uint16_t* w = w_uv + static_cast<int64_t>(h) * dv * dc;
    for (int i = wid; i < dv; i += nw) {
        const uint16_t* wr = w + static_cast<int64_t>(i) * dc;
        float acc[kUvGroups];
#pragma unroll
        for (int gg = 0; gg < kUvGroups; ++gg) acc[gg] = 0.f;
        for (int j = lane; j < dc; j += 32) {
            const float wv = bf16_to_f32(wr[j]);
#pragma unroll
            for (int gg = 0; gg < kUvGroups; ++gg) acc[gg] = fmaf(wv, ol[gg * dc + j], acc[gg]);
        }
#pragma unroll
        for (int gg = 0; gg < kUvGroups; ++gg) {
            const float v = warp_sum(acc[gg]);
            if (lane == 0 && gg < ng)
                out[(static_cast<int64_t>(g0 + gg) * H + h) * dv + i] = f32_to_bf16(v);
        }
    }
}

}  // namespace mla
