// Tensor-core versions of the small GEMMs around the attention (used when the
// sizes are multiples of the tile: see tc_gemm_dims_ok in the ABI):
//   absorb:    Q[g, h, 0:d_c] = bf16(q_nope[g, h] W_UK[h]),  Q[g, h, d_c:] = q_pe[g, h]
//              (query absorption, "MLA架构：低秩注意力机制优化LLM显存与计算效率" 3.1)
//   merge+UV:  the split-KV partials of (g, h) merged into o_lat (log-sum-exp
//              weights), then out[g, h] = bf16(W_UV[h] o_lat[g, h])
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
    pdl_wait();
    pdl_trigger();
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

// -------------------------------------------------- merge + up-projection
// Log-sum-exp merge of the split partials fused with the value up-projection:
//   o_lat[g, h] = sum_i w_i o_i / sum_i w_i,  w_i = exp(lse_i - max_i lse_i)
//   out[g, h, :] = bf16(W_UV[h] o_lat[g, h])
// Partial i of (g, h) is o_part[i, h, :] (PartT: float, or bf16 bits in
// uint16_t), already divided by its own softmax denominator; parts with
// lse = -inf weigh 0 and a group without a finite part gives zeros. o_lat is
// rounded to bf16 in shared memory (the GEMM's A operand) while W_UV[h]
// streams in. grid (H, ceil(G / 64)); block 256; dynamic smem uv_tc_smem(dc, dv).
__host__ __device__ inline size_t uv_tc_smem(int dc, int dv) {
    return sizeof(uint16_t) * (static_cast<size_t>(kTcRows) + dv) * (dc + 8);
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const uint16_t* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
    v[4] = __uint_as_float(u.z << 16); v[5] = __uint_as_float(u.z & 0xffff0000u);
    v[6] = __uint_as_float(u.w << 16); v[7] = __uint_as_float(u.w & 0xffff0000u);
}

template <typename PartT>
__global__ void __launch_bounds__(kTcThreads) merge_uv_tc_kernel(
    const PartT* __restrict__ o_part, const float* __restrict__ lse_part, const int32_t* __restrict__ part_offsets,
    const uint16_t* __restrict__ w_uv, int32_t G, int32_t H, int32_t dc, int32_t dv, uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint16_t sm_uv[];
    const int ld = dc + 8;
    uint16_t* As = sm_uv;               // [64][dc + 8]  o_lat rows of head h (bf16)
    uint16_t* Bs = As + kTcRows * ld;   // [dv][dc + 8]  W_UV[h] (latent column contiguous)
    const int h = blockIdx.x, g0 = blockIdx.y * kTcRows;
    const int c8s = dc / 8;
    for (int i = threadIdx.x; i < dv * c8s; i += blockDim.x) {
        const int n = i / c8s, c8 = (i % c8s) * 8;
        wmma16::cp_async16(Bs + n * ld + c8, w_uv + (static_cast<int64_t>(h) * dv + n) * dc + c8);
    }
    wmma16::cp_async_commit();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows_used = min(kTcRows, G - g0);
    // merge: one warp per group row; lane l owns columns 256 j + 8 l .. +7
    constexpr int kMaxJ = 2;  // dc <= 512
    for (int r = warp; r < kTcRows; r += kTcThreads / 32) {
        uint16_t* dst = As + r * ld;
        float acc[kMaxJ][8];
#pragma unroll
        for (int j = 0; j < kMaxJ; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
        float den = 0.f;
        if (r < rows_used) {
            const int32_t g = g0 + r;
            const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
            float M = -INFINITY;
            for (int32_t p = p0 + lane; p < p1; p += 32) M = fmaxf(M, lse_part[static_cast<int64_t>(p) * H + h]);
            M = warp_max(M);
            if (M != -INFINITY) {
#pragma unroll 4
                for (int32_t p = p0; p < p1; ++p) {
                    const float l = lse_part[static_cast<int64_t>(p) * H + h];
                    const float w = l == -INFINITY ? 0.f : __expf(l - M);
                    den += w;
                    const PartT* src = o_part + (static_cast<int64_t>(p) * H + h) * dc;
#pragma unroll
                    for (int j = 0; j < kMaxJ; ++j) {
                        const int col = 256 * j + 8 * lane;
                        if (col < dc) {
                            float v[8];
                            load8(src + col, v);
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[j][e] = fmaf(w, v[e], acc[j][e]);
                        }
                    }
                }
            }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
        for (int j = 0; j < kMaxJ; ++j) {
            const int col = 256 * j + 8 * lane;
            if (col < dc)
                *reinterpret_cast<uint4*>(dst + col) =
                    make_uint4(pack_bf16x2(acc[j][0] * inv, acc[j][1] * inv), pack_bf16x2(acc[j][2] * inv, acc[j][3] * inv),
                               pack_bf16x2(acc[j][4] * inv, acc[j][5] * inv), pack_bf16x2(acc[j][6] * inv, acc[j][7] * inv));
        }
    }
    wmma16::cp_async_wait<0>();
    __syncthreads();
    for (int wt = warp; wt < 4 * (dv / 64); wt += kTcThreads / 32) {
        const int r0 = 16 * (wt & 3), c0 = 64 * (wt >> 2);
        if (r0 >= rows_used) continue;  // an all-zero row block
        float accg[8][4] = {};
        for (int k0 = 0; k0 < dc; k0 += 16) wmma16::warp_tile_k16<true>(accg, As, ld, r0, Bs, ld, c0, k0);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = c0 + 8 * nt + 2 * (lane & 3);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int g = g0 + r0 + (lane >> 2) + 8 * hf;
                if (g < G)
                    *reinterpret_cast<uint32_t*>(out + (static_cast<int64_t>(g) * H + h) * dv + col) =
                        pack_bf16x2(accg[nt][2 * hf], accg[nt][2 * hf + 1]);
            }
        }
    }
}

}  // namespace mla
