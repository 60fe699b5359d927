// tcgen05 versions of the per-head GEMMs around the attention, for DeepSeek-V3
// like dims (their weights are read once per step, so they are bandwidth
// bound: operands arrive by TMA in 128-byte-swizzled boxes, one CTA of four
// warps per head and block of up to 128 new tokens, accumulators in TMEM):
//   absorb: Q[g, h, 0:d_c] = bf16(q_nope[g, h] W_UK[h]),  Q[g, h, d_c:] = q_pe[g, h]
//           (query absorption, "MLA架构：低秩注意力机制优化LLM显存与计算效率" 3.1)
//   UV:     out[g, h] = bf16(W_UV[h] o_lat[g, h])
// and the log-sum-exp merge of the split-KV partials into bf16 o_lat that
// feeds the UV GEMM.
//
// Roles (128 threads): lane 0 of warp 0 issues the TMA loads, lane 0 of
// warp 1 the MMAs (M = 128 token rows, cta_group::1), warp 2 owns the TMEM
// allocation, and all four warps (thread t = TMEM lane t = token row g0 + t)
// run the epilogue. Every mbarrier wait is bounded (ptx::mbar_wait).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace tc05 {

constexpr int kRows = 128;     // token rows per CTA (the MMA's M)
constexpr int kThreads = 128;
constexpr int kBoxBytes = 64 * 2;  // one swizzled 64-column bf16 row

__device__ __forceinline__ uint32_t bar_addr(uint8_t* smem, int off, int i) {
    return ptx::smem_u32(smem + off + 8 * i);
}

// ---------------------------------------------------------------- merge
// o_lat[g, h, :] = sum_i w_i o_part[i, h, :] / sum_i w_i over the partials i
// of group g (part_offsets[g] .. part_offsets[g+1]-1), w_i = exp(lse_i - max
// lse); parts with lse = -inf weigh 0, a group without a finite part gives
// zeros. One warp per (g, h); d_c is 256 or 512. grid (G, ceil(H / 4)); block 128.
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
__global__ void __launch_bounds__(128) merge_kernel(const PartT* __restrict__ o_part,
                                                    const float* __restrict__ lse_part,
                                                    const int32_t* __restrict__ part_offsets, int32_t G, int32_t H,
                                                    int32_t dc, uint16_t* __restrict__ o_lat) {
    pdl_wait();
    pdl_trigger();
    // lane l owns columns 16 l .. 16 l + 15 (d_c = 512); the weights of up to 32
    // parts are computed by the lanes at once, and the part rows are loaded four
    // at a time before they are used, so a warp waits on few memory round trips.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x, h = blockIdx.y * 4 + warp;
    if (h >= H) return;
    const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
    float M = -INFINITY;
    for (int32_t p = p0 + lane; p < p1; p += 32) M = fmaxf(M, lse_part[static_cast<int64_t>(p) * H + h]);
    M = warp_max(M);
    const int ncol = dc / 32;  // columns per lane: 16 for d_c = 512, 8 for 256
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int32_t c0 = p0; c0 < p1; c0 += 32) {
            const int32_t pl = c0 + lane;
            const float l = pl < p1 ? lse_part[static_cast<int64_t>(pl) * H + h] : -INFINITY;
            const float wl = l == -INFINITY ? 0.f : __expf(l - M);
            den += warp_sum(wl);
            const int n = min(32, p1 - c0);
            for (int i0 = 0; i0 < n; i0 += 4) {
                float v[4][16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (i0 + u < n) {
                        const PartT* src = o_part + (static_cast<int64_t>(c0 + i0 + u) * H + h) * dc + ncol * lane;
                        float (&v0)[8] = *reinterpret_cast<float(*)[8]>(&v[u][0]);
                        float (&v1)[8] = *reinterpret_cast<float(*)[8]>(&v[u][8]);
                        load8(src, v0);
                        if (ncol == 16) load8(src + 8, v1);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float w = __shfl_sync(0xffffffffu, wl, (i0 + u) & 31);
                    if (i0 + u < n) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (e < ncol) acc[e] = fmaf(w, v[u][e], acc[e]);
                    }
                }
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint16_t* dst = o_lat + (static_cast<int64_t>(g) * H + h) * dc + ncol * lane;
#pragma unroll
    for (int k = 0; k < 2; ++k)
        if (8 * k < ncol)
            *reinterpret_cast<uint4*>(dst + 8 * k) = make_uint4(
                pack_bf16x2(acc[8 * k] * inv, acc[8 * k + 1] * inv), pack_bf16x2(acc[8 * k + 2] * inv, acc[8 * k + 3] * inv),
                pack_bf16x2(acc[8 * k + 4] * inv, acc[8 * k + 5] * inv), pack_bf16x2(acc[8 * k + 6] * inv, acc[8 * k + 7] * inv));
}

// ------------------------------------------------------------------- UV
// out[g, h, :] = bf16(W_UV[h] o_lat[g, h, :]) for g in [g0, g0 + 128).
// tm_ol: o_lat as 2-D [G rows, H * d_c columns], box {64, 128}; tm_w: W_UV as
// 2-D [H * d_v rows, d_c columns], box {64, d_v}; both 128-byte swizzled and
// K-major (the latent index is the contraction). The d_c / 64 K-blocks
// stream through a ring of kUvStages stages (A box + B box each).
// grid (H, ceil(G / 128)); block 128; dynamic smem uv_smem(d_v).
constexpr int kUvStages = 4;

__host__ __device__ inline int uv_stage_bytes(int dv) { return kRows * kBoxBytes + dv * kBoxBytes; }
__host__ __device__ inline size_t uv_smem(int dv) {
    return static_cast<size_t>(kUvStages) * uv_stage_bytes(dv) + 256 + 1024;
}

__global__ void __launch_bounds__(kThreads, 1) uv_kernel(const __grid_constant__ CUtensorMap tm_ol,
                                                        const __grid_constant__ CUtensorMap tm_w, int32_t G,
                                                        int32_t H, int32_t dc, int32_t dv,
                                                        uint16_t* __restrict__ out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int stage_bytes = uv_stage_bytes(dv);
    const int off_bar = kUvStages * stage_bytes;  // full[s], empty[s], done
    volatile int* abort = reinterpret_cast<volatile int*>(smem + off_bar + 8 * (2 * kUvStages + 1));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * kUvStages + 1) + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, g0 = blockIdx.y * kRows;
    const int nk = dc / 64;
    if (threadIdx.x == 0) {
        *abort = 0;
        for (int s = 0; s < kUvStages; ++s) {
            ptx::mbar_init(bar_addr(smem, off_bar, s), 1);
            ptx::mbar_init(bar_addr(smem, off_bar, kUvStages + s), 1);
        }
        ptx::mbar_init(bar_addr(smem, off_bar, 2 * kUvStages), 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_ol);
        ptx::prefetch_tmap(&tm_w);
    }
    if (warp == 2) {
        ptx::tmem_alloc_1(ptx::smem_u32(tmem_slot), dv <= 32 ? 32 : dv <= 64 ? 64 : dv <= 128 ? 128 : 256);
        ptx::tmem_relinquish_1();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();
    pdl_trigger();

    if (warp == 0 && lane == 0) {  // producer
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kUvStages;
            if (!ptx::mbar_wait(bar_addr(smem, off_bar, kUvStages + s), ((kb / kUvStages) & 1) ^ 1, abort)) break;
            const uint32_t full = bar_addr(smem, off_bar, s);
            const uint32_t dst = ptx::smem_u32(smem + s * stage_bytes);
            ptx::mbar_arrive_expect_tx_local(full, stage_bytes);
            ptx::tma_load_2d(dst, &tm_ol, h * dc + 64 * kb, g0, full);
            ptx::tma_load_2d(dst + kRows * kBoxBytes, &tm_w, 64 * kb, h * dv, full);
        }
    } else if (warp == 1 && lane == 0) {  // MMA issuer
        const uint32_t idesc = ptx::idesc_bf16(kRows, dv, false, false);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kUvStages;
            if (!ptx::mbar_wait(bar_addr(smem, off_bar, s), (kb / kUvStages) & 1, abort)) break;
            ptx::tc_fence_after();
            const uint32_t base = ptx::smem_u32(smem + s * stage_bytes);
            const uint64_t da = ptx::smem_desc_sw128(base, 16, 1024);
            const uint64_t db = ptx::smem_desc_sw128(base + kRows * kBoxBytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) ptx::mma_bf16_1(tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
            ptx::mma_commit_1(bar_addr(smem, off_bar, kUvStages + s));
        }
        ptx::mma_commit_1(bar_addr(smem, off_bar, 2 * kUvStages));
    }
    // epilogue: thread t = TMEM lane t = token row g0 + t
    const bool ok = ptx::mbar_wait(bar_addr(smem, off_bar, 2 * kUvStages), 0, abort);
    ptx::tc_fence_after();
    if (ok) {
        const int g = g0 + static_cast<int>(threadIdx.x);
        const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        for (int c0 = 0; c0 < dv; c0 += 32) {
            float v[32];
            ptx::tmem_ld32(tl + c0, v);
            ptx::tmem_wait_ld();
            if (g < G) {
                uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(g) * H + h) * dv + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(ptx::bf16x2(v[8 * i], v[8 * i + 1]), ptx::bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                        ptx::bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                        ptx::bf16x2(v[8 * i + 6], v[8 * i + 7]));
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_1(tmem, dv <= 32 ? 32 : dv <= 64 ? 64 : dv <= 128 ? 128 : 256);
    }
}

// --------------------------------------------------------------- absorb
// Q[g, h, 0:d_c] = bf16(q_nope[g, h, :] W_UK[h]) and Q[g, h, d_c:] = q_pe[g, h]
// for g in [g0, g0 + 128). tm_q: q_nope as 2-D [G rows, H * d_n columns], box
// {64, 128} (K-major A); tm_w: W_UK as 2-D [H * d_n rows, d_c columns], box
// {64, d_n} (MN-major B: the latent index is contiguous). All d_n / 64 A boxes
// and d_c / 64 B boxes are loaded at once (d_n = 128, d_c = 512: 160 KB), then
// the (d_c / 256) x (d_n / 16) MMAs of N = 256 run into d_c TMEM columns.
// grid (H, ceil(G / 128)); block 128; dynamic smem absorb_smem(d_n, d_c).
__host__ __device__ inline size_t absorb_a_bytes(int dn) { return static_cast<size_t>(dn / 64) * kRows * kBoxBytes; }
__host__ __device__ inline size_t absorb_smem(int dn, int dc) {
    return absorb_a_bytes(dn) + static_cast<size_t>(dc / 64) * dn * kBoxBytes + 256 + 1024;
}

__global__ void __launch_bounds__(kThreads, 1) absorb_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_w,
                                                            const uint16_t* __restrict__ q_pe, int32_t G,
                                                            int32_t H, int32_t dn, int32_t dc, int32_t dr,
                                                            uint16_t* __restrict__ q_out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int a_bytes = static_cast<int>(absorb_a_bytes(dn));
    const int b_box = dn * kBoxBytes;  // one [d_n x 64] box of W_UK[h]
    const int off_bar = a_bytes + (dc / 64) * b_box;  // full, done
    volatile int* abort = reinterpret_cast<volatile int*>(smem + off_bar + 16);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 32);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, g0 = blockIdx.y * kRows;
    if (threadIdx.x == 0) {
        *abort = 0;
        ptx::mbar_init(bar_addr(smem, off_bar, 0), 1);
        ptx::mbar_init(bar_addr(smem, off_bar, 1), 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_w);
    }
    if (warp == 2) {
        ptx::tmem_alloc_1(ptx::smem_u32(tmem_slot), 512);
        ptx::tmem_relinquish_1();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();
    pdl_trigger();
    const uint32_t full = bar_addr(smem, off_bar, 0), done = bar_addr(smem, off_bar, 1);

    if (warp == 0 && lane == 0) {  // producer: everything at once
        ptx::mbar_arrive_expect_tx_local(full, a_bytes + (dc / 64) * b_box);
        for (int kb = 0; kb < dn / 64; ++kb)
            ptx::tma_load_2d(ptx::smem_u32(smem + kb * kRows * kBoxBytes), &tm_q, h * dn + 64 * kb, g0, full);
        for (int nb = 0; nb < dc / 64; ++nb)
            ptx::tma_load_2d(ptx::smem_u32(smem + a_bytes + nb * b_box), &tm_w, 64 * nb, h * dn, full);
    } else if (warp == 1 && lane == 0) {  // MMA issuer
        constexpr uint32_t idesc = ptx::idesc_bf16(kRows, 256, false, true);
        if (ptx::mbar_wait(full, 0, abort)) {
            ptx::tc_fence_after();
            const uint32_t sa = ptx::smem_u32(smem), sb = ptx::smem_u32(smem + a_bytes);
            for (int nh = 0; nh < dc / 256; ++nh) {
                // B: rows (k) 16 ks .. +15 = two 8-row atoms (2 KB), columns 256 nh .. +255 = 4 boxes (LBO = box)
                const uint64_t db = ptx::smem_desc_sw128(sb + 4 * nh * b_box, b_box, 1024);
                for (int ks = 0; ks < dn / 16; ++ks) {
                    const uint64_t da = ptx::smem_desc_sw128(sa + (ks >> 2) * kRows * kBoxBytes, 16, 1024) +
                                        static_cast<uint64_t>(2 * (ks & 3));
                    ptx::mma_bf16_1(tmem + 256 * nh, da, db + static_cast<uint64_t>((2048 * ks) >> 4), idesc,
                                    ks != 0);
                }
            }
        }
        ptx::mma_commit_1(done);
    }
    // epilogue: thread t = TMEM lane t = token row g0 + t
    const bool ok = ptx::mbar_wait(done, 0, abort);
    ptx::tc_fence_after();
    if (ok) {
        const int g = g0 + static_cast<int>(threadIdx.x);
        const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int D = dc + dr;
        for (int c0 = 0; c0 < dc; c0 += 32) {
            float v[32];
            ptx::tmem_ld32(tl + c0, v);
            ptx::tmem_wait_ld();
            if (g < G) {
                uint4* dst = reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(g) * H + h) * D + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(ptx::bf16x2(v[8 * i], v[8 * i + 1]), ptx::bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                        ptx::bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                        ptx::bf16x2(v[8 * i + 6], v[8 * i + 7]));
            }
        }
        if (g < G) {  // the RoPE part of the query row
            const uint4* src = reinterpret_cast<const uint4*>(q_pe + (static_cast<int64_t>(g) * H + h) * dr);
            uint4* dst = reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(g) * H + h) * D + dc);
            for (int i = 0; i < dr / 8; ++i) dst[i] = src[i];
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_1(tmem, 512);
    }
}

}  // namespace tc05
}  // namespace mla
