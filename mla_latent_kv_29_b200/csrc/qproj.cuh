// Query projection of new tokens ("MLA架构：低秩注意力机制优化LLM显存与计算效率"
// 2.1 and 1): c_q = RMSNorm(x . W_qa) (q_a_proj, q_a_layernorm), q = c_q . W_qb
// (q_b_proj), each head's qk_head_dim values split into the d_n non-RoPE part
// and the d_r RoPE part, the latter rotated (rotate-half RoPE of
// "一次讲透MHA、GQA、MQA、MLA", "MLA的实现") at the token's position.
// The two GEMMs run on tc05::row_gemm_kernel; the kernels here are the row
// normalisation between them and, for RoPE widths other than 64, the split +
// RoPE after them (with 64 the second GEMM writes the heads itself).
// Both run once per CTA, so their loops stay rolled.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kQNormThreads = 256;
constexpr int kQNormCols = 8;  // q_rank <= 256 * 8

// out[t, :] = bf16(c / sqrt(mean(c^2) + eps) * gamma), c = sum over the
// `splits` partials part[z][t][:] (fp32, [splits][T][R]). grid T; block 256;
// dynamic smem 4 R bytes.
__global__ void __launch_bounds__(kQNormThreads) q_norm_kernel(const float* __restrict__ part, int32_t splits,
                                                              int32_t T, int32_t R,
                                                              const uint16_t* __restrict__ gamma, float eps,
                                                              uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float row[];
    __shared__ float red[kQNormThreads / 32];
    const int t = blockIdx.x;
    // thread j owns columns j + 256 i (i < kQNormCols); the columns of four
    // splits are requested together, so four splits cost one memory round trip
    float acc[kQNormCols];
#pragma unroll
    for (int i = 0; i < kQNormCols; ++i) acc[i] = 0.f;
    const int64_t zs = static_cast<int64_t>(T) * R;
    const float* src = part + static_cast<int64_t>(t) * R + threadIdx.x;
#pragma unroll 1
    for (int z0 = 0; z0 < splits; z0 += 4) {
        float v[4][kQNormCols];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int i = 0; i < kQNormCols; ++i)
                v[u][i] = (z0 + u < splits && static_cast<int>(threadIdx.x) + kQNormThreads * i < R)
                              ? __ldg(src + (z0 + u) * zs + kQNormThreads * i)
                              : 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int i = 0; i < kQNormCols; ++i) acc[i] += v[u][i];
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kQNormCols; ++i) {
        const int n = static_cast<int>(threadIdx.x) + kQNormThreads * i;
        if (n < R) {
            row[n] = acc[i];
            ss = fmaf(acc[i], acc[i], ss);
        }
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < kQNormThreads / 32 ? red[threadIdx.x] : 0.f;
        v = warp_sum(v);
        if (threadIdx.x == 0) red[0] = rsqrtf(v / static_cast<float>(R) + eps);
    }
    __syncthreads();
    const float r = red[0];
#pragma unroll 1
    for (int n = threadIdx.x; n < R; n += kQNormThreads) {
        float c = row[n] * r;
        if (gamma) c *= bf16_to_f32(gamma[n]);
        out[static_cast<int64_t>(t) * R + n] = f32_to_bf16(c);
    }
}

// Rotation frequencies of the RoPE part, base^(-2i/d_r), computed on the host
// in double precision (d_r <= 2 kQMaxRopePairs).
constexpr int kQMaxRopePairs = 64;
struct QSplitParams {
    const float* part;  // [splits][T][H * (d_n + d_r)] fp32
    const int32_t* positions;
    uint16_t* q_nope;   // [T][H][d_n]
    uint16_t* q_pe;     // [T][H][d_r]
    int32_t splits, T, H, dn, dr;
    double inv_freq[kQMaxRopePairs];
};

// Thread j of CTA (t, h): j < d_n copies q[t, h, j] to q_nope; j = d_n + i
// (i < d_r / 2) rotates the pair (i, i + d_r / 2) of the RoPE part by
// positions[t] * inv_freq[i]. grid (T, H); block >= d_n + d_r / 2, a
// multiple of 32.
__global__ void q_split_rope_kernel(const __grid_constant__ QSplitParams P) {
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
    const int D = P.dn + P.dr, half = P.dr / 2;
    const int64_t N = static_cast<int64_t>(P.H) * D;
    auto q_at = [&](int col) {
        float v = 0.f;
#pragma unroll 1
        for (int z = 0; z < P.splits; ++z) v += P.part[(static_cast<int64_t>(z) * P.T + t) * N + h * D + col];
        return v;
    };
    if (j < P.dn) {
        P.q_nope[(static_cast<int64_t>(t) * P.H + h) * P.dn + j] = f32_to_bf16(q_at(j));
    } else if (j < P.dn + half) {
        const int i = j - P.dn;
        // angle formed in double and reduced to [-pi, pi] with a two-term 2 pi, so
        // that the float sine and cosine stay on their short-argument path
        const double angle = static_cast<double>(P.positions[t]) * P.inv_freq[i];
        const double k = rint(angle * 0.15915494309189535);  // 1 / (2 pi)
        const double reduced = fma(-k, 2.4492935982947064e-16, fma(-k, 6.283185307179586, angle));
        float s, c;
        sincosf(static_cast<float>(reduced), &s, &c);
        const float x1 = q_at(P.dn + i), x2 = q_at(P.dn + i + half);
        uint16_t* dst = P.q_pe + (static_cast<int64_t>(t) * P.H + h) * P.dr;
        dst[i] = f32_to_bf16(x1 * c - x2 * s);
        dst[i + half] = f32_to_bf16(x2 * c + x1 * s);
    }
}

}  // namespace mla
