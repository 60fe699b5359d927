// Tensor-core versions of the small GEMMs around the attention (used when the
// sizes are multiples of the tile: see tc_gemm_dims_ok in the ABI):
//   absorb:    Q[g, h, 0:d_c] = bf16(q_nope[g, h] W_UK[h]),  Q[g, h, d_c:] = q_pe[g, h]
//              (query absorption, "MLA架构：低秩注意力机制优化LLM显存与计算效率" 3.1)
//   merge:     the split-KV partials of (g, h) into bf16 o_lat (log-sum-exp weights)
//   UV:        out[g, h] = bf16(W_UV[h] o_lat[g, h])
//   append:    split-K partial sums of x . W_kva (kv_a_proj_with_mqa, 2.2)
// Each loads its weight tile once per CTA and runs 16 x 64 warp tiles.
#pragma once

#include "common.cuh"
#include "combine.cuh"
#include "warp_mma.cuh"

namespace mla {

constexpr int kTcRows = 64;    // token rows per CTA
constexpr int kTcThreads = 256;

// ---------------------------------------------------------------- absorb
// grid (H, dc / 128, ceil(G / 64)); dynamic smem absorb_tc_smem(dn).
__host__ __device__ inline size_t absorb_tc_smem(int dn) {
    return sizeof(uint16_t) * (static_cast<size_t>(kTcRows) * (dn + 8) + static_cast<size_t>(dn) * (128 + 8));
}

__global__ void __launch_bounds__(kTcThreads) absorb_tc_kernel(
    const uint16_t* __restrict__ q_nope, const uint16_t* __restrict__ q_pe, const uint16_t* __restrict__ w_uk,
    uint16_t* __restrict__ q_out, int32_t G, int32_t H, int32_t dn, int32_t dc, int32_t dr) {
    extern __shared__ __align__(16) uint16_t sm_abs[];
    const int lda = dn + 8, ldb = 128 + 8;
    uint16_t* As = sm_abs;                   // [64][dn + 8]   q_nope rows
    uint16_t* Bs = As + kTcRows * lda;       // [dn][136]      W_UK[h][:, n0:n0+128]
    const int h = blockIdx.x, n0 = blockIdx.y * 128, g0 = blockIdx.z * kTcRows;
    const int D = dc + dr;
    for (int i = threadIdx.x; i < dn * 16; i += blockDim.x) {
        const int k = i >> 4, c8 = (i & 15) * 8;
        wmma16::cp_async16(Bs + k * ldb + c8, w_uk + (static_cast<int64_t>(h) * dn + k) * dc + n0 + c8);
    }
    for (int i = threadIdx.x; i < kTcRows * (dn / 8); i += blockDim.x) {
        const int r = i / (dn / 8), c8 = (i % (dn / 8)) * 8;
        const int g = g0 + r;
        if (g < G)
            wmma16::cp_async16(As + r * lda + c8, q_nope + (static_cast<int64_t>(g) * H + h) * dn + c8);
        else
            *reinterpret_cast<uint4*>(As + r * lda + c8) = make_uint4(0u, 0u, 0u, 0u);
    }
    wmma16::cp_async_commit();
    if (blockIdx.y == 0) {  // the RoPE part of the query row
        for (int i = threadIdx.x; i < kTcRows * dr; i += blockDim.x) {
            const int r = i / dr, k = i % dr, g = g0 + r;
            if (g < G)
                q_out[(static_cast<int64_t>(g) * H + h) * D + dc + k] = q_pe[(static_cast<int64_t>(g) * H + h) * dr + k];
        }
    }
    wmma16::cp_async_wait<0>();
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = 16 * (warp & 3), c0 = 64 * (warp >> 2);
    float acc[8][4] = {};
    for (int k0 = 0; k0 < dn; k0 += 16) wmma16::warp_tile_k16<false>(acc, As, lda, r0, Bs, ldb, c0, k0);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int col = n0 + c0 + 8 * nt + 2 * (lane & 3);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int g = g0 + r0 + (lane >> 2) + 8 * hf;
            if (g < G)
                *reinterpret_cast<uint32_t*>(q_out + (static_cast<int64_t>(g) * H + h) * D + col) =
                    pack_bf16x2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
        }
    }
}

// ------------------------------------------------------------------ merge
// Log-sum-exp merge of the split partials of (g, h) into o_lat[g, h] (bf16):
// one warp per (group, head); lane l owns latent columns 4l + 128j .. +3.
// grid (G, ceil(H / 8)); block 256.
__global__ void __launch_bounds__(256) merge_bf16_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part, const int32_t* __restrict__ part_offsets,
    int32_t G, int32_t H, int32_t dc, uint16_t* __restrict__ o_lat) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x, h = blockIdx.y * 8 + warp;
    if (h >= H) return;
    const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
    float M = -INFINITY;
    for (int32_t p = p0 + lane; p < p1; p += 32) M = fmaxf(M, lse_part[static_cast<int64_t>(p) * H + h]);
    M = warp_max(M);
    const int nj = dc / 128;  // float4 column groups per lane (4 for d_c = 512)
    float4 acc[4] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f),
                     make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    float den = 0.f;
    if (M != -INFINITY) {
#pragma unroll 2
        for (int32_t p = p0; p < p1; ++p) {
            const float l = lse_part[static_cast<int64_t>(p) * H + h];
            const float w = l == -INFINITY ? 0.f : __expf(l - M);
            den += w;
            const float4* src = reinterpret_cast<const float4*>(o_part + (static_cast<int64_t>(p) * H + h) * dc) + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < nj) {
                    const float4 u = src[32 * j];
                    acc[j].x = fmaf(w, u.x, acc[j].x); acc[j].y = fmaf(w, u.y, acc[j].y);
                    acc[j].z = fmaf(w, u.z, acc[j].z); acc[j].w = fmaf(w, u.w, acc[j].w);
                }
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint16_t* dst = o_lat + (static_cast<int64_t>(g) * H + h) * dc + 4 * lane;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (j < nj)
            *reinterpret_cast<uint2*>(dst + 128 * j) =
                make_uint2(pack_bf16x2(acc[j].x * inv, acc[j].y * inv), pack_bf16x2(acc[j].z * inv, acc[j].w * inv));
}

// ------------------------------------------------------------ up-projection
// out[g, h, :] = bf16(W_UV[h] o_lat[g, h, :]); grid (H, ceil(G / 64)); block 256;
// dynamic smem uv_tc_smem(dc, dv).
__host__ __device__ inline size_t uv_tc_smem(int dc, int dv) {
    return sizeof(uint16_t) * (static_cast<size_t>(kTcRows) + dv) * (dc + 8);
}

__global__ void __launch_bounds__(kTcThreads) uv_tc_kernel(const uint16_t* __restrict__ o_lat,
                                                            const uint16_t* __restrict__ w_uv, int32_t G, int32_t H,
                                                            int32_t dc, int32_t dv, uint16_t* __restrict__ out) {
    extern __shared__ __align__(16) uint16_t sm_uv[];
    const int ld = dc + 8;
    uint16_t* As = sm_uv;               // [64][dc + 8]  o_lat rows of head h
    uint16_t* Bs = As + kTcRows * ld;   // [dv][dc + 8]  W_UV[h] (latent column contiguous)
    const int h = blockIdx.x, g0 = blockIdx.y * kTcRows;
    const int c8s = dc / 8;
    for (int i = threadIdx.x; i < dv * c8s; i += blockDim.x) {
        const int n = i / c8s, c8 = (i % c8s) * 8;
        wmma16::cp_async16(Bs + n * ld + c8, w_uv + (static_cast<int64_t>(h) * dv + n) * dc + c8);
    }
    for (int i = threadIdx.x; i < kTcRows * c8s; i += blockDim.x) {
        const int r = i / c8s, c8 = (i % c8s) * 8, g = g0 + r;
        if (g < G)
            wmma16::cp_async16(As + r * ld + c8, o_lat + (static_cast<int64_t>(g) * H + h) * dc + c8);
        else
            *reinterpret_cast<uint4*>(As + r * ld + c8) = make_uint4(0u, 0u, 0u, 0u);
    }
    wmma16::cp_async_commit();
    wmma16::cp_async_wait<0>();
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows_used = min(kTcRows, G - g0);
    for (int wt = warp; wt < 4 * (dv / 64); wt += kTcThreads / 32) {
        const int r0 = 16 * (wt & 3), c0 = 64 * (wt >> 2);
        if (r0 >= rows_used) continue;  // an all-zero row block
        float acc[8][4] = {};
        for (int k0 = 0; k0 < dc; k0 += 16) wmma16::warp_tile_k16<true>(acc, As, ld, r0, Bs, ld, c0, k0);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = c0 + 8 * nt + 2 * (lane & 3);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int g = g0 + r0 + (lane >> 2) + 8 * hf;
                if (g < G)
                    *reinterpret_cast<uint32_t*>(out + (static_cast<int64_t>(g) * H + h) * dv + col) =
                        pack_bf16x2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
            }
        }
    }
}

// ----------------------------------------------------------------- append
// part[z][t][n] = sum over split z's K range of x[t][k] * w[k][n].
// grid (N / 64, ceil(T / 64), splits); block 128 (4 warps x 16 rows);
// K range per split a multiple of 64; 2-stage cp.async pipeline over 64-wide K chunks.
constexpr int kApTc = 64;
constexpr int kApTcLd = kApTc + 8;

__global__ void __launch_bounds__(128) append_gemm_tc_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, float* __restrict__ part,
    int32_t T, int32_t K, int32_t N, int32_t k_per_split) {
    __shared__ __align__(16) uint16_t As[2][kApTc * kApTcLd];  // [t][k]
    __shared__ __align__(16) uint16_t Bs[2][kApTc * kApTcLd];  // [k][n]
    const int n0 = blockIdx.x * kApTc, t0 = blockIdx.y * kApTc;
    const int k_begin = blockIdx.z * k_per_split;
    const int k_end = min(K, k_begin + k_per_split);
    const int nchunks = k_end > k_begin ? (k_end - k_begin) / kApTc : 0;
    auto load = [&](int chunk, int buf) {
        const int k0 = k_begin + chunk * kApTc;
        for (int i = threadIdx.x; i < kApTc * 8; i += 128) {
            const int r = i >> 3, c8 = (i & 7) * 8;
            const int t = t0 + r;
            if (t < T)
                wmma16::cp_async16(&As[buf][r * kApTcLd + c8], x + static_cast<int64_t>(t) * K + k0 + c8);
            else
                *reinterpret_cast<uint4*>(&As[buf][r * kApTcLd + c8]) = make_uint4(0u, 0u, 0u, 0u);
            wmma16::cp_async16(&Bs[buf][r * kApTcLd + c8], w + static_cast<int64_t>(k0 + r) * N + n0 + c8);
        }
        wmma16::cp_async_commit();
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[8][4] = {};
    if (nchunks > 0) load(0, 0);
    for (int ch = 0; ch < nchunks; ++ch) {
        if (ch + 1 < nchunks) {
            load(ch + 1, (ch + 1) & 1);
            wmma16::cp_async_wait<1>();
        } else {
            wmma16::cp_async_wait<0>();
        }
        __syncthreads();
#pragma unroll
        for (int k0 = 0; k0 < kApTc; k0 += 16)
            wmma16::warp_tile_k16<false>(acc, As[ch & 1], kApTcLd, 16 * warp, Bs[ch & 1], kApTcLd, 0, k0);
        __syncthreads();
    }
    float* dst = part + static_cast<int64_t>(blockIdx.z) * T * N;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int col = n0 + 8 * nt + 2 * (lane & 3);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int t = t0 + 16 * warp + (lane >> 2) + 8 * hf;
            if (t < T)
                *reinterpret_cast<float2*>(dst + static_cast<int64_t>(t) * N + col) =
                    make_float2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
        }
    }
}

}  // namespace mla
