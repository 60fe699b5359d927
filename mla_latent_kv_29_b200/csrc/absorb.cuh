// Query absorption ("matrix absorption" of the key up-projection into the
// query; "MLA架构：低秩注意力机制优化LLM显存与计算效率" section 3.1, and the
// absorbed forward of "一次讲透MHA、GQA、MQA、MLA" section "MLA的实现"):
//   Q[g, h, 0:d_c]       = bf16( W_UK[h]^T q_nope[g, h] )
//   Q[g, h, d_c:d_c+d_r] = q_pe[g, h]
// Q is the packed per-head query row the decode kernels read: it has the
// same 576-wide (c_kv ++ k_pe) layout as a cache row.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kAbsorbThreads = 256;
constexpr int kAbsorbGroups = 32;  // groups per CTA (weights are read once per CTA)

// grid (H, ceil(G / kAbsorbGroups)); dynamic smem kAbsorbGroups * dn floats.
__global__ void __launch_bounds__(kAbsorbThreads) absorb_q_kernel(
    const uint16_t* __restrict__ q_nope, const uint16_t* __restrict__ q_pe,
    const uint16_t* __restrict__ w_uk, uint16_t* __restrict__ q_out,
    int32_t G, int32_t H, int32_t dn, int32_t dc, int32_t dr) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float qn[];  // [kAbsorbGroups][dn]
    const int h = blockIdx.x;
    const int g0 = blockIdx.y * kAbsorbGroups;
    const int ng = min(kAbsorbGroups, G - g0);
    const int row = dc + dr;
    for (int i = threadIdx.x; i < ng * dn; i += blockDim.x) {
        const int gg = i / dn, k = i - gg * dn;
        qn[i] = bf16_to_f32(q_nope[(static_cast<int64_t>(g0 + gg) * H + h) * dn + k]);
    }
    // copy the RoPE part of the query
    for (int i = threadIdx.x; i < ng * dr; i += blockDim.x) {
        const int gg = i / dr, k = i - gg * dr;
        q_out[(static_cast<int64_t>(g0 + gg) * H + h) * row + dc + k] =
            q_pe[(static_cast<int64_t>(g0 + gg) * H + h) * dr + k];
    }
    __syncthreads();
    const uint16_t* w = w_uk + static_cast<int64_t>(h) * dn * dc;
    for (int j = threadIdx.x; j < dc; j += blockDim.x) {
        float acc[kAbsorbGroups];
#pragma unroll
        for (int gg = 0; gg < kAbsorbGroups; ++gg) acc[gg] = 0.f;
        for (int k = 0; k < dn; ++k) {
            const float wv = bf16_to_f32(w[static_cast<int64_t>(k) * dc + j]);
#pragma unroll
            for (int gg = 0; gg < kAbsorbGroups; ++gg) acc[gg] = fmaf(qn[gg * dn + k], wv, acc[gg]);
        }
#pragma unroll
        for (int gg = 0; gg < kAbsorbGroups; ++gg)
            if (gg < ng) q_out[(static_cast<int64_t>(g0 + gg) * H + h) * row + j] = f32_to_bf16(acc[gg]);
    }
}

}  // namespace mla
