// tcgen05 versions of the GEMMs around the attention, for DeepSeek-V3 like
// dims (their weights are read once per step, so they are bandwidth bound:
// operands arrive by TMA in 128-byte-swizzled boxes, accumulators in TMEM):
//   absorb:     Q[g, h, 0:d_c] = bf16(q_nope[g, h] W_UK[h]),  Q[g, h, d_c:] = q_pe[g, h]
//               (query absorption, "MLA架构：低秩注意力机制优化LLM显存与计算效率" 3.1)
//   merge + UV: out[g, h] = bf16(W_UV[h] o_lat[g, h]) with o_lat the
//               log-sum-exp merge of the split-KV partials, merged on chip
//               (merge_uv_kernel), or merged into memory (merge_kernel) and
//               then multiplied (uv_kernel)
//   row GEMM:   y = x W (fp32 partials over K ranges) for x [T, K] and W
//               [K, N] (row_gemm_kernel): the cache append's x W_kva, the
//               query projection's x W_qa and c_q W_qb (the latter, with one
//               K range, writing q_nope and the rotated q_pe itself), and the
//               output projection (sum_partials_kernel adds its partials into
//               bf16).
//
// Roles of the 128-thread kernels: lane 0 of warp 0 issues the TMA loads,
// lane 0 of warp 1 the MMAs (M = 128, cta_group::1), warp 2 owns the TMEM
// allocation, and all four warps (thread t = TMEM lane t = row t of the MMA)
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
    // Lane l owns columns ncol * l .. + ncol - 1. The lse values of up to 32 parts
    // (one per lane) and the rows of four parts are requested together, so a group
    // with at most four parts costs one memory round trip; more parts follow four
    // rows at a time, their weights taken from the lanes by shuffles.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x, h = blockIdx.y * 4 + warp;
    if (h >= H) return;
    const int32_t p0 = part_offsets[g], p1 = part_offsets[g + 1];
    const int ncol = dc / 32;  // columns per lane: 16 for d_c = 512, 8 for 256
    auto load_row = [&](int32_t p, float (&v)[16]) {
        const PartT* src = o_part + (static_cast<int64_t>(p) * H + h) * dc + ncol * lane;
        float (&v0)[8] = *reinterpret_cast<float(*)[8]>(&v[0]);
        float (&v1)[8] = *reinterpret_cast<float(*)[8]>(&v[8]);
        load8(src, v0);
        if (ncol == 16) load8(src + 8, v1);
    };
    float v[4][16];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (p0 + u < p1) load_row(p0 + u, v[u]);
    float lse_first = p0 + lane < p1 ? lse_part[static_cast<int64_t>(p0 + lane) * H + h] : -INFINITY;
    float M = lse_first;
    for (int32_t p = p0 + 32 + lane; p < p1; p += 32) M = fmaxf(M, lse_part[static_cast<int64_t>(p) * H + h]);
    M = warp_max(M);
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int32_t c0 = p0; c0 < p1; c0 += 32) {
            const float l = c0 == p0 ? lse_first
                                     : (c0 + lane < p1 ? lse_part[static_cast<int64_t>(c0 + lane) * H + h] : -INFINITY);
            const float wl = l == -INFINITY ? 0.f : __expf(l - M);
            den += warp_sum(wl);
            const int n = min(32, p1 - c0);
            for (int i0 = 0; i0 < n; i0 += 4) {
                if (c0 != p0 || i0 != 0) {  // the first four rows are already in flight
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (i0 + u < n) load_row(c0 + i0 + u, v[u]);
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
    // warp-uniform (the tensor-memory loads below are warp-collective)
    const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_addr(smem, off_bar, 2 * kUvStages), 0, abort));
    ptx::tc_fence_after();
    if (ok) {
        const int g = g0 + static_cast<int>(threadIdx.x);
        const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
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

// ------------------------------------------------------------ merge + UV
// out[g, h, :] = bf16(W_UV[h] o_lat[g, h, :]) for the kMuvRows groups g of
// block blockIdx.y, where o_lat[g, h] is the log-sum-exp merge of group g's
// bf16 split-KV partials (the merge_kernel rule, rounded to bf16). o_lat
// never goes to memory: the product is taken transposed, D[d, g] = sum_c
// W_UV[h][d, c] o_lat[g, c], with M = d_v = 128 rows of W_UV[h] (A) and
// N = 64 groups (B), so a small batch pads no MMA row, and each 64-column
// block kb of B is merged straight into shared memory, in the 128-byte
// swizzled K-major layout, from the partial rows of the block's groups.
// The CTA's groups own the consecutive partial slots [P0, P1); per block kb a
// ring stage receives, by TMA, W_UV[h][:, 64 kb ..] (box {64, 128} of tm_w =
// W_UV as 2-D [H * d_v rows, d_c columns]) and the slots' columns 64 kb ..
// (n_box boxes {64 columns, 1 head, 64 slots} of tm_p = the partials as 3-D
// [slots][H][d_c]), so the stages are in flight together and no warp waits
// on a chain of dependent loads. Warp 8 is the producer: it refills the stage
// of block kb with block kb + 4 as soon as block kb's MMAs are done, so no
// merge warp waits on an MMA. The weights exp(lse - max) / sum come first:
// the slots' lse into shared memory in one round trip, then a thread (or, for
// fewer than 32 groups, a warp) per group. Merge thread t merges group t / 4,
// columns 16 (t % 4) .. + 15 of a block; thread 0 issues the MMAs.
// grid (H, ceil(G / 64)); block 288; dynamic smem merge_uv_smem(n_box);
// d_v = 128, d_c a multiple of 64 up to 512, P1 - P0 <= 64 n_box, n_box <= 4.
constexpr int kMuvThreads = 288;       // 8 merge warps + 1 producer warp
constexpr int kMuvMergeThreads = 256;
constexpr int kMuvRows = 64;     // groups per CTA (the MMA's N)
constexpr int kMuvDv = 128;      // the MMA's M
constexpr int kMuvStages = 4;
constexpr int kMuvMaxBox = 4;    // slot boxes of 64 per stage at most
constexpr int kMuvSlotBox = 64 * kBoxBytes;  // 8 KB: 64 slots x 64 columns
__device__ __forceinline__ void merge_sync() {  // the 8 merge warps only (named barrier 1)
    asm volatile("bar.sync 1, %0;" ::"n"(kMuvMergeThreads) : "memory");
}
__host__ __device__ inline int merge_uv_stage_bytes(int n_box) {
    return n_box * kMuvSlotBox + kMuvDv * kBoxBytes + kMuvRows * kBoxBytes;
}
__host__ __device__ inline size_t merge_uv_smem(int n_box) {
    return static_cast<size_t>(kMuvStages) * merge_uv_stage_bytes(n_box) + 256 + 512 + 4 * 64 * kMuvMaxBox + 1024;
}

__global__ void __launch_bounds__(kMuvThreads, 1) merge_uv_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                                 const __grid_constant__ CUtensorMap tm_p,
                                                                 const float* __restrict__ lse_part,
                                                                 const int32_t* __restrict__ part_offsets,
                                                                 int32_t G, int32_t H, int32_t dc, int32_t n_box,
                                                                 uint16_t* __restrict__ out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int nk = dc / 64;
    const int stage_bytes = merge_uv_stage_bytes(n_box);
    const int off_w = n_box * kMuvSlotBox, off_bm = off_w + kMuvDv * kBoxBytes;  // within a stage
    const int off_bar = kMuvStages * stage_bytes;  // full[s], empty[s], done
    volatile int* abort = reinterpret_cast<volatile int*>(smem + off_bar + 8 * (2 * kMuvStages + 1));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * kMuvStages + 1) + 16);
    int32_t* offs = reinterpret_cast<int32_t*>(smem + off_bar + 256);          // kMuvRows + 1 entries
    float* wgt = reinterpret_cast<float*>(smem + off_bar + 256 + 512);         // per slot of [P0, P1)
    const int t = static_cast<int>(threadIdx.x), warp = t >> 5, lane = t & 31;
    const bool producer = warp == kMuvMergeThreads / 32;
    const int h = blockIdx.x, g0 = blockIdx.y * kMuvRows;
    const int R = min(kMuvRows, G - g0);
    if (t == 0) {
        *abort = 0;
        for (int i = 0; i <= 2 * kMuvStages; ++i) ptx::mbar_init(bar_addr(smem, off_bar, i), 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_w);
        ptx::prefetch_tmap(&tm_p);
    }
    if (warp == 2) {
        ptx::tmem_alloc_1(ptx::smem_u32(tmem_slot), kMuvRows);
        ptx::tmem_relinquish_1();
    }
    // part_offsets come from the plan launch, which finished before the attention
    // launch (this one's predecessor) could pass its own dependency wait
    if (t <= R) offs[t] = part_offsets[g0 + t];
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int32_t P0 = offs[0], NP = offs[R] - P0;
    const int nb = NP > 0 ? (NP + 63) / 64 : 0;  // slot boxes this CTA needs
    const bool fits = nb <= n_box;
    if (!fits && t == 0) record_status(MLA_ERR_DEVICE_FAULT);
    const uint32_t stage_tx = fits ? static_cast<uint32_t>(nb * kMuvSlotBox + kMuvDv * kBoxBytes)
                                   : static_cast<uint32_t>(kMuvDv * kBoxBytes);
    auto load_w = [&](int kb, uint32_t full) {
        ptx::tma_load_2d(ptx::smem_u32(smem + (kb % kMuvStages) * stage_bytes + off_w), &tm_w, 64 * kb, h * kMuvDv,
                         full);
    };
    auto load_slots = [&](int kb, uint32_t full) {
        if (!fits) return;
        for (int b = 0; b < nb; ++b)
            ptx::tma_load_3d(ptx::smem_u32(smem + (kb % kMuvStages) * stage_bytes + b * kMuvSlotBox), &tm_p, 64 * kb, h,
                             P0 + 64 * b, full);
    };
    if (producer && lane == 0) {  // the weights are not written by earlier launches: request them now
        for (int kb = 0; kb < min(nk, kMuvStages); ++kb) {
            ptx::mbar_arrive_expect_tx_local(bar_addr(smem, off_bar, kb), stage_tx);
            load_w(kb, bar_addr(smem, off_bar, kb));
        }
    }
    pdl_wait();
    pdl_trigger();

    if (producer) {
        // ---- producer: the slots of the first stages, then each later block into the
        // stage its block kb - 4 leaves once that block's MMAs are done
        if (lane == 0) {
            for (int kb = 0; kb < min(nk, kMuvStages); ++kb) load_slots(kb, bar_addr(smem, off_bar, kb));
            for (int kb = kMuvStages; kb < nk; ++kb) {
                const int st = kb % kMuvStages;
                if (!ptx::mbar_wait(bar_addr(smem, off_bar, kMuvStages + st), ((kb / kMuvStages) - 1) & 1, abort))
                    break;
                const uint32_t full = bar_addr(smem, off_bar, st);
                ptx::mbar_arrive_expect_tx_local(full, stage_tx);
                load_w(kb, full);
                load_slots(kb, full);
            }
        }
    } else {
        // ---- weights (merge warps). This code runs once per CTA, so it is kept short
        // (loops, not unrolled copies): on a cold instruction cache every new line of
        // code costs a round trip to L2. (1) every slot's lse into shared memory.
        if (fits)
            for (int i = t; i < NP; i += kMuvMergeThreads) wgt[i] = lse_part[static_cast<int64_t>(P0 + i) * H + h];
        merge_sync();
        // (2) per group: max, sum, then the normalised weights in place. Many groups:
        // a thread each; few (long groups, small batches): a warp each, lanes over slots.
        if (fits && R >= 32) {
            if (t < R) {
                const int32_t a = offs[t] - P0, b = offs[t + 1] - P0;
                float M = -INFINITY;
                for (int32_t i = a; i < b; ++i) M = fmaxf(M, wgt[i]);
                float den = 0.f;
                if (M != -INFINITY)
                    for (int32_t i = a; i < b; ++i) den += wgt[i] == -INFINITY ? 0.f : __expf(wgt[i] - M);
                const float inv = den > 0.f ? __fdividef(1.f, den) : 0.f;
                for (int32_t i = a; i < b; ++i) {
                    const float l = wgt[i];
                    wgt[i] = l == -INFINITY || M == -INFINITY ? 0.f : __expf(l - M) * inv;
                }
            }
        } else if (fits) {
#pragma unroll 1
            for (int jj = warp; jj < R; jj += kMuvMergeThreads / 32) {
                const int32_t a = offs[jj] - P0, b = offs[jj + 1] - P0;
                float M = -INFINITY;
                for (int32_t i = a + lane; i < b; i += 32) M = fmaxf(M, wgt[i]);
                M = warp_max(M);
                float den = 0.f;
                if (M != -INFINITY)
                    for (int32_t i = a + lane; i < b; i += 32) den += wgt[i] == -INFINITY ? 0.f : __expf(wgt[i] - M);
                den = warp_sum(den);
                const float inv = den > 0.f ? __fdividef(1.f, den) : 0.f;
                for (int32_t i = a + lane; i < b; i += 32) {  // each lane rewrites only the slots it read
                    const float l = wgt[i];
                    wgt[i] = l == -INFINITY || M == -INFINITY ? 0.f : __expf(l - M) * inv;
                }
            }
        }
        merge_sync();

        // ---- per 64-column block: merge into B, then 4 MMAs (thread 0)
        const int j = t >> 2, q = t & 3;
        const int32_t s0 = j < R ? offs[j] - P0 : 0, s1 = j < R ? offs[j + 1] - P0 : 0;
#pragma unroll 1
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % kMuvStages;
            uint8_t* stage = smem + st * stage_bytes;
            const bool ok = ptx::mbar_wait(bar_addr(smem, off_bar, st), (kb / kMuvStages) & 1, abort);
            if (j < R) {
                float acc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = 0.f;
                if (ok && fits) {
#pragma unroll 1
                    for (int32_t i = s0; i < s1; ++i) {  // slot i: box i / 64, swizzled row i % 64
                        const float w = wgt[i];
                        const uint8_t* row = stage + (i >> 6) * kMuvSlotBox + (i & 63) * kBoxBytes;
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const uint4 u = *reinterpret_cast<const uint4*>(row + (((2 * q + c) ^ (i & 7)) << 4));
                            const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                acc[8 * c + 2 * k] = fmaf(w, __uint_as_float(x[k] << 16), acc[8 * c + 2 * k]);
                                acc[8 * c + 2 * k + 1] =
                                    fmaf(w, __uint_as_float(x[k] & 0xffff0000u), acc[8 * c + 2 * k + 1]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    *reinterpret_cast<uint4*>(stage + off_bm + j * kBoxBytes + (((2 * q + c) ^ (j & 7)) << 4)) =
                        make_uint4(ptx::bf16x2(acc[8 * c], acc[8 * c + 1]), ptx::bf16x2(acc[8 * c + 2], acc[8 * c + 3]),
                                   ptx::bf16x2(acc[8 * c + 4], acc[8 * c + 5]),
                                   ptx::bf16x2(acc[8 * c + 6], acc[8 * c + 7]));
            }
            ptx::fence_proxy_async_smem();  // B was written through the generic proxy
            merge_sync();
            if (t == 0) {
                ptx::tc_fence_after();
                constexpr uint32_t idesc = ptx::idesc_bf16(kMuvDv, kMuvRows, false, false);
                const uint64_t da = ptx::smem_desc_sw128(ptx::smem_u32(stage + off_w), 16, 1024);
                const uint64_t db = ptx::smem_desc_sw128(ptx::smem_u32(stage + off_bm), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) ptx::mma_bf16_1(tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
                ptx::mma_commit_1(bar_addr(smem, off_bar, kMuvStages + st));
            }
        }
        if (t == 0) ptx::mma_commit_1(bar_addr(smem, off_bar, 2 * kMuvStages));
    }
    __syncwarp();
    __syncthreads();

    // ---- epilogue: thread t < 128 = TMEM lane t = output column d; TMEM column j = group g0 + j.
    // D goes through shared memory (stage 0, free once every MMA is done) as bf16 [64 groups][128]
    // so that the stores are whole 16-byte pieces of the output rows.
    const bool done =
        __all_sync(0xffffffffu, ptx::mbar_wait(bar_addr(smem, off_bar, 2 * kMuvStages), 0, abort) && !*abort);
    ptx::tc_fence_after();
    uint16_t* stg = reinterpret_cast<uint16_t*>(smem);
    if (warp < 4) {
#pragma unroll 1
        for (int c0 = 0; c0 < R; c0 += 32) {
            float v[32];
            ptx::tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) stg[(c0 + i) * kMuvDv + t] = static_cast<uint16_t>(ptx::bf16x2(v[i], 0.f) & 0xffffu);
        }
    }
    __syncthreads();
    if (done) {
        for (int idx = t; idx < R * (kMuvDv / 8); idx += kMuvThreads) {
            const int jj = idx / (kMuvDv / 8), c8 = idx % (kMuvDv / 8);
            *reinterpret_cast<uint4*>(out + (static_cast<int64_t>(g0 + jj) * H + h) * kMuvDv + 8 * c8) =
                *reinterpret_cast<const uint4*>(stg + jj * kMuvDv + 8 * c8);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_1(tmem, kMuvRows);
    }
}

// --------------------------------------------------------------- absorb
// Q[g, h, 256 z .. 256 z + 255] = bf16(q_nope[g, h, :] W_UK[h][:, 256 z ..]) for
// g in [g0, g0 + 128), and (z = 0) Q[g, h, d_c:] = q_pe[g, h]. tm_q: q_nope as
// 2-D [G rows, H * d_n columns], box {64, 128} (K-major A); tm_w: W_UK as 2-D
// [H * d_n rows, d_c columns], box {64, d_n} (MN-major B: the latent index is
// contiguous). Each CTA loads its d_n / 64 A boxes and the 4 B boxes of its
// 256 output columns at once (d_n = 128: 96 KB, two CTAs per SM), then runs
// d_n / 16 MMAs of N = 256 into 256 TMEM columns. With q_f16 set, Q is written
// as IEEE half instead of bf16 (q_pe converted too): the operand type of the
// attention over the FP8 cache, whose MMAs run on f16.
// grid (H, ceil(G / 128), d_c / 256); block 128; dynamic smem absorb_smem(d_n).
__host__ __device__ inline size_t absorb_a_bytes(int dn) { return static_cast<size_t>(dn / 64) * kRows * kBoxBytes; }
__host__ __device__ inline size_t absorb_smem(int dn) {
    return absorb_a_bytes(dn) + static_cast<size_t>(4) * dn * kBoxBytes + 256 + 1024;
}

__global__ void __launch_bounds__(kThreads) absorb_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                          const __grid_constant__ CUtensorMap tm_w,
                                                          const uint16_t* __restrict__ q_pe, int32_t G, int32_t H,
                                                          int32_t dn, int32_t dc, int32_t dr,
                                                          uint16_t* __restrict__ q_out, int32_t q_f16) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int a_bytes = static_cast<int>(absorb_a_bytes(dn));
    const int b_box = dn * kBoxBytes;  // one [d_n x 64] box of W_UK[h]
    const int off_bar = a_bytes + 4 * b_box;  // full, done
    volatile int* abort = reinterpret_cast<volatile int*>(smem + off_bar + 16);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 32);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, g0 = blockIdx.y * kRows, z = blockIdx.z;
    if (threadIdx.x == 0) {
        *abort = 0;
        ptx::mbar_init(bar_addr(smem, off_bar, 0), 1);
        ptx::mbar_init(bar_addr(smem, off_bar, 1), 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_w);
    }
    if (warp == 2) {
        ptx::tmem_alloc_1(ptx::smem_u32(tmem_slot), 256);
        ptx::tmem_relinquish_1();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // This kernel reads only the caller's inputs and writes only the query region
    // of the workspace. It follows the plan launch, which started it only after its
    // own dependency wait (so all earlier work is complete) and which it does not
    // read: the whole kernel runs beside the plan, and its dependency wait comes
    // last, so that its completion still implies the plan's.
    pdl_trigger();
    const uint32_t full = bar_addr(smem, off_bar, 0), done = bar_addr(smem, off_bar, 1);

    if (warp == 0 && lane == 0) {  // producer: everything at once
        ptx::mbar_arrive_expect_tx_local(full, a_bytes + 4 * b_box);
        for (int kb = 0; kb < dn / 64; ++kb)
            ptx::tma_load_2d(ptx::smem_u32(smem + kb * kRows * kBoxBytes), &tm_q, h * dn + 64 * kb, g0, full);
        for (int nb = 0; nb < 4; ++nb)
            ptx::tma_load_2d(ptx::smem_u32(smem + a_bytes + nb * b_box), &tm_w, 256 * z + 64 * nb, h * dn, full);
    } else if (warp == 1 && lane == 0) {  // MMA issuer
        constexpr uint32_t idesc = ptx::idesc_bf16(kRows, 256, false, true);
        if (ptx::mbar_wait(full, 0, abort)) {
            ptx::tc_fence_after();
            const uint32_t sa = ptx::smem_u32(smem), sb = ptx::smem_u32(smem + a_bytes);
            // B: rows (k) 16 ks .. +15 = two 8-row atoms (2 KB), the 4 boxes of 64 columns LBO apart
            const uint64_t db = ptx::smem_desc_sw128(sb, b_box, 1024);
            for (int ks = 0; ks < dn / 16; ++ks) {
                const uint64_t da = ptx::smem_desc_sw128(sa + (ks >> 2) * kRows * kBoxBytes, 16, 1024) +
                                    static_cast<uint64_t>(2 * (ks & 3));
                ptx::mma_bf16_1(tmem, da, db + static_cast<uint64_t>((2048 * ks) >> 4), idesc, ks != 0);
            }
        }
        ptx::mma_commit_1(done);
    }
    // epilogue: thread t = TMEM lane t = token row g0 + t. The RoPE part of the
    // query row (CTAs with z = 0) is requested before the wait for the MMAs.
    const int g = g0 + static_cast<int>(threadIdx.x);
    constexpr int kPe = 8;  // d_r / 8 uint4 pieces, d_r <= 64 on this path
    uint4 pe[kPe];
    const bool copy_pe = g < G && z == 0;
    if (copy_pe) {
        const uint4* src = reinterpret_cast<const uint4*>(q_pe + (static_cast<int64_t>(g) * H + h) * dr);
#pragma unroll
        for (int i = 0; i < kPe; ++i)
            if (i < dr / 8) pe[i] = src[i];
    }
    const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(done, 0, abort));  // warp-uniform
    ptx::tc_fence_after();
    if (ok) {
        const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int D = dc + dr;
#pragma unroll 1  // one-shot code: kept short for a cold instruction cache
        for (int c0 = 0; c0 < 256; c0 += 32) {
            float v[32];
            ptx::tmem_ld32(tl + c0, v);
            ptx::tmem_wait_ld();
            if (g < G) {
                uint4* dst = reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(g) * H + h) * D + 256 * z + c0);
                if (q_f16) {  // f16 queries for the FP8 cache's f16 MMAs
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(ptx::f16x2(v[8 * i], v[8 * i + 1]), ptx::f16x2(v[8 * i + 2], v[8 * i + 3]),
                                            ptx::f16x2(v[8 * i + 4], v[8 * i + 5]),
                                            ptx::f16x2(v[8 * i + 6], v[8 * i + 7]));
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(ptx::bf16x2(v[8 * i], v[8 * i + 1]), ptx::bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                            ptx::bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                            ptx::bf16x2(v[8 * i + 6], v[8 * i + 7]));
                }
            }
        }
        if (copy_pe) {  // the RoPE part of the query row (as f16 when q_f16)
            uint4* dst = reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(g) * H + h) * D + dc);
#pragma unroll
            for (int i = 0; i < kPe; ++i) {
                if (i >= dr / 8) continue;
                uint4 u = pe[i];
                if (q_f16) {
                    auto cv = [](uint32_t w) {
                        return ptx::f16x2(bf16_to_f32(w & 0xFFFFu), bf16_to_f32(w >> 16));
                    };
                    u = make_uint4(cv(u.x), cv(u.y), cv(u.z), cv(u.w));
                }
                dst[i] = u;
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_1(tmem, 256);
    }
    pdl_wait();
}

// --------------------------------------------------------------- row GEMM
// part[z][t][n0 .. n0 + 64 nb - 1] = x[t, K-range z] W[K-range z, n0 .. n0 + 64 nb - 1]
// (fp32) for t in [m0, m0 + 128): a GEMM with few rows (new tokens) whose cost
// is streaming the weight W once. Used for the joint down-projection of the
// cache append (kv_a_proj_with_mqa, "MLA架构：低秩注意力机制优化LLM显存与计算效率"
// 2.2), the query projections (2.1) and the output projection. The grid covers
// the weight with (column tile of 64 nb, K-range of k_per_cta blocks of 64)
// work units sized so that whole waves of CTAs stream it; the consumer (the
// append or query epilogue, or sum_partials_kernel) sums the Z partials of a
// column tile, requesting four at a time.
// Each CTA streams its K-blocks through a ring of stages (x box {64, 128 rows}
// plus nb W boxes {64 columns, 64 rows}) into an M 128 x N 64 nb TMEM
// accumulator and stores its rows of the partial tile.
// tm_x: x as 2-D [T rows, K columns]; tm_w: W as 2-D [K rows, N columns], box
// {64, 64} (MN-major B). grid (N / (64 nb), ceil(T / 128), Z); block 128;
// dynamic smem row_gemm_smem(nb).
constexpr int kRgSmemBudget = 200 * 1024;
__host__ __device__ inline int row_gemm_stage_bytes(int nb) { return kRows * kBoxBytes + nb * 64 * kBoxBytes; }
__host__ __device__ inline int row_gemm_stages(int nb) { return kRgSmemBudget / row_gemm_stage_bytes(nb); }
__host__ __device__ inline size_t row_gemm_smem(int nb) {
    return static_cast<size_t>(row_gemm_stages(nb)) * row_gemm_stage_bytes(nb) + 256 + 1024;
}

// The query projection's second product can write its heads directly: with
// one K-range (no partials), 64-column RoPE parts and d_n a multiple of 64,
// every 64-column piece of a tile is one piece of one head, either of its
// non-RoPE part (rounded to bf16 into q_nope) or its whole RoPE part (rotate-
// half pairs (i, i + 32), both in the thread's registers, rotated by
// positions[t] * inv_freq[i] and rounded into q_pe).
struct QHeadOut {
    const int32_t* positions;  // null: the kernel stores fp32 partials instead
    uint16_t* q_nope;          // [T, H, d_n]
    uint16_t* q_pe;            // [T, H, 64]
    int32_t dn;
    double inv_freq[32];       // base^(-2i/64), computed on the host in double
};

__global__ void __launch_bounds__(kThreads, 1) row_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                              const __grid_constant__ CUtensorMap tm_w, int32_t T,
                                                              int32_t N, int32_t k_blocks, int32_t k_per_cta,
                                                              int32_t nb, float* __restrict__ part,
                                                              const __grid_constant__ QHeadOut qo) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int stage_bytes = row_gemm_stage_bytes(nb), n_stages = row_gemm_stages(nb);
    const int off_bar = n_stages * stage_bytes;  // full[s], empty[s], done
    volatile int* abort = reinterpret_cast<volatile int*>(smem + off_bar + 8 * (2 * n_stages + 1));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * n_stages + 1) + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ncols = 64 * nb;
    const int n0 = blockIdx.x * ncols, m0 = blockIdx.y * kRows, z = blockIdx.z;
    part += static_cast<int64_t>(z) * T * N;
    const int kb0 = z * k_per_cta;
    const int nk = max(0, min(k_per_cta, k_blocks - kb0));  // this CTA's K-blocks of 64
    if (threadIdx.x == 0) {
        *abort = 0;
        for (int i = 0; i < n_stages; ++i) {
            ptx::mbar_init(bar_addr(smem, off_bar, i), 1);
            ptx::mbar_init(bar_addr(smem, off_bar, n_stages + i), 1);
        }
        ptx::mbar_init(bar_addr(smem, off_bar, 2 * n_stages), 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_x);
        ptx::prefetch_tmap(&tm_w);
    }
    if (warp == 2) {
        ptx::tmem_alloc_1(ptx::smem_u32(tmem_slot), ncols);
        ptx::tmem_relinquish_1();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {  // producer
        // The weights are not written by earlier launches: the first stages' weight
        // boxes are requested before the dependency wait, the activations after it.
        const int pre = min(nk, n_stages);
        for (int i = 0; i < pre; ++i) {
            const uint32_t full = bar_addr(smem, off_bar, i);
            const uint32_t dst = ptx::smem_u32(smem + i * stage_bytes);
            ptx::mbar_arrive_expect_tx_local(full, stage_bytes);
            for (int b = 0; b < nb; ++b)
                ptx::tma_load_2d(dst + (kRows + 64 * b) * kBoxBytes, &tm_w, n0 + 64 * b, 64 * (kb0 + i), full);
        }
        pdl_wait();
        pdl_trigger();
        for (int i = 0; i < pre; ++i)
            ptx::tma_load_2d(ptx::smem_u32(smem + i * stage_bytes), &tm_x, 64 * (kb0 + i), m0,
                             bar_addr(smem, off_bar, i));
        for (int i = pre; i < nk; ++i) {
            const int st = i % n_stages;
            if (!ptx::mbar_wait(bar_addr(smem, off_bar, n_stages + st), ((i / n_stages) & 1) ^ 1, abort)) break;
            const uint32_t full = bar_addr(smem, off_bar, st);
            const uint32_t dst = ptx::smem_u32(smem + st * stage_bytes);
            ptx::mbar_arrive_expect_tx_local(full, stage_bytes);
            ptx::tma_load_2d(dst, &tm_x, 64 * (kb0 + i), m0, full);
            for (int b = 0; b < nb; ++b)
                ptx::tma_load_2d(dst + (kRows + 64 * b) * kBoxBytes, &tm_w, n0 + 64 * b, 64 * (kb0 + i), full);
        }
    } else {
        pdl_wait();
        pdl_trigger();
        if (warp == 1 && lane == 0) {  // MMA issuer
            const uint32_t idesc = ptx::idesc_bf16(kRows, ncols, false, true);
            for (int i = 0; i < nk; ++i) {
                const int st = i % n_stages;
                if (!ptx::mbar_wait(bar_addr(smem, off_bar, st), (i / n_stages) & 1, abort)) break;
                ptx::tc_fence_after();
                const uint32_t base = ptx::smem_u32(smem + st * stage_bytes);
                const uint64_t da = ptx::smem_desc_sw128(base, 16, 1024);
                // B: the nb boxes of 64 columns are 8 KB apart (LBO); 8-row atoms 1 KB apart (SBO)
                const uint64_t db = ptx::smem_desc_sw128(base + kRows * kBoxBytes, 64 * kBoxBytes, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_bf16_1(tmem, da + 2 * kk, db + static_cast<uint64_t>((2048 * kk) >> 4), idesc,
                                    (i | kk) != 0);
                ptx::mma_commit_1(bar_addr(smem, off_bar, n_stages + st));
            }
            ptx::mma_commit_1(bar_addr(smem, off_bar, 2 * n_stages));
        }
    }
    // epilogue: thread t = TMEM lane t = token row m0 + t, 32 columns at a time
    const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_addr(smem, off_bar, 2 * n_stages), 0, abort));
    ptx::tc_fence_after();
    const int t = static_cast<int>(threadIdx.x);
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if (qo.positions) {  // the head split: each 64-column piece of the tile is one piece of one head
        const int D = qo.dn + 64, H = N / D;
        const int64_t row = m0 + t;
#pragma unroll 1
        for (int pc = 0; pc < nb; ++pc) {
            float v[64];
            {
                float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
                float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
                ptx::tmem_ld32(tl + 64 * pc, v0);
                ptx::tmem_ld32(tl + 64 * pc + 32, v1);
                ptx::tmem_wait_ld();
            }
            if (!ok || nk == 0) {
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = 0.f;
            }
            const int n = n0 + 64 * pc;
            const int h = n / D, off = n - h * D;
            if (row >= T) continue;
            uint4* dst;
            if (off < qo.dn) {
                dst = reinterpret_cast<uint4*>(qo.q_nope + (row * H + h) * qo.dn + off);
            } else {
                dst = reinterpret_cast<uint4*>(qo.q_pe + (row * H + h) * 64);
                const double pos = static_cast<double>(qo.positions[row]);
#pragma unroll 1
                for (int i = 0; i < 32; ++i) {
                    // angle reduced to [-pi, pi] in double with a two-term 2 pi, so that the
                    // float sine and cosine stay on their short-argument path
                    const double angle = pos * qo.inv_freq[i];
                    const double k = rint(angle * 0.15915494309189535);  // 1 / (2 pi)
                    const double reduced = fma(-k, 2.4492935982947064e-16, fma(-k, 6.283185307179586, angle));
                    float sn, cs;
                    sincosf(static_cast<float>(reduced), &sn, &cs);
                    const float x1 = v[i], x2 = v[i + 32];
                    v[i] = x1 * cs - x2 * sn;
                    v[i + 32] = x2 * cs + x1 * sn;
                }
            }
#pragma unroll
            for (int c = 0; c < 8; ++c)
                dst[c] = make_uint4(ptx::bf16x2(v[8 * c], v[8 * c + 1]), ptx::bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                    ptx::bf16x2(v[8 * c + 4], v[8 * c + 5]), ptx::bf16x2(v[8 * c + 6], v[8 * c + 7]));
        }
    }
#pragma unroll 1
    for (int c0 = 0; c0 < (qo.positions ? 0 : ncols); c0 += 32) {
        float v[32];
        ptx::tmem_ld32(tl + c0, v);
        ptx::tmem_wait_ld();
        if (!ok || nk == 0) {  // nothing accumulated (or a wait gave up): contribute zeros
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        if (m0 + t < T) {
            float4* dst = reinterpret_cast<float4*>(part + static_cast<int64_t>(m0 + t) * N + n0 + c0);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_1(tmem, ncols);
    }
}

// y[t, :] = bf16(sum_z part[z][t][:]) for the row GEMM's Z partials ([Z][T][N]
// fp32, N a multiple of 4). Thread = 4 consecutive columns of one row; up to
// four partials are requested before any is summed. grid ceil(T N / 512);
// block 128.
__global__ void __launch_bounds__(128) sum_partials_kernel(const float* __restrict__ part, int32_t Z, int32_t T,
                                                           int32_t N, uint16_t* __restrict__ y) {
    pdl_wait();
    pdl_trigger();
    const int64_t i4 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    const int64_t zs = static_cast<int64_t>(T) * N;
    if (i4 >= zs) return;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int z0 = 0; z0 < Z; z0 += 4) {
        float4 b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            b[u] = z0 + u < Z ? __ldg(reinterpret_cast<const float4*>(part + (z0 + u) * zs + i4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) { a.x += b[u].x; a.y += b[u].y; a.z += b[u].z; a.w += b[u].w; }
    }
    *reinterpret_cast<uint2*>(y + i4) = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
}

}  // namespace tc05
}  // namespace mla
