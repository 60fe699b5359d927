// Split-KV absorbed decode on CUDA cores, for any supported dims.
//
// Per (worker, head block) CTA and per segment of the split-KV schedule:
// scores z_t = scale * (q_lat . c_t + q_pe . k_pe_t) over the segment's
// tokens (the absorbed score of "一次讲透MHA、GQA、MQA、MLA", section
// "MLA的实现"), an online softmax, o = sum_t p_t c_t, and a normalised partial
// (o / l, lse = m + ln l) written to the segment's slot. The softmax weights
// are rounded to bf16 before the value sum, as the tensor-core kernel does.
#pragma once

#include "common.cuh"
#include "plan.cuh"

namespace mla {

constexpr int kGenThreads = 256;
constexpr int kGenHeads = 16;   // heads per CTA
constexpr int kGenTokens = 32;  // tokens per sub-tile (= schedule tile)
constexpr int kGenMaxCols = 32; // dc <= 16 * kGenMaxCols

struct GenericDecodeParams {
    const uint16_t* q;       // [G, H, D] bf16, D = dc + dr (q_lat ++ q_pe)
    const uint16_t* pool;    // [num_blocks * bs, D] bf16
    const int32_t* block_table;
    const int32_t* context_lens;
    const PlanHeader* hdr;
    const int32_t* worker_group;
    const int32_t* tile_prefix;
    const int32_t* part_offsets;
    float* o_part;           // [n_parts, H, dc]
    float* lse_part;         // [n_parts, H]
    int64_t num_blocks;
    int32_t batch, max_blocks_per_seq, block_size, q_len, H, dc, dr;
    float scale;
};

// grid (workers, ceil(H / kGenHeads)); block 256; dynamic smem from generic_decode_smem().
__host__ __device__ inline size_t generic_decode_smem(int dc, int dr) {
    const int D = dc + dr, Dp = D + 1;
    return sizeof(float) * (static_cast<size_t>(kGenHeads) * Dp + static_cast<size_t>(kGenTokens) * Dp +
                            kGenHeads * kGenTokens + 4 * kGenHeads);
}

__global__ void __launch_bounds__(kGenThreads) generic_decode_kernel(GenericDecodeParams P) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float sm[];
    const int D = P.dc + P.dr, Dp = D + 1;
    float* sq = sm;                              // [kGenHeads][Dp]
    float* skv = sq + kGenHeads * Dp;            // [kGenTokens][Dp]
    float* ss = skv + kGenTokens * Dp;           // [kGenHeads][kGenTokens]
    float* s_m = ss + kGenHeads * kGenTokens;    // running max
    float* s_l = s_m + kGenHeads;                // running sum
    float* s_a = s_l + kGenHeads;                // rescale factor of this sub-tile

    const int tid = threadIdx.x;
    const int h0 = blockIdx.y * kGenHeads;
    const int hl = tid / 16;                  // local head owned in the PV stage
    const int cl = tid % 16;                  // column phase
    const int ncol = (P.dc + 15) / 16;

    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kGenTokens, blockIdx.x);
    Segment seg;
    while (it.next(seg)) {
        const int32_t g = seg.group;
        const int32_t b = g / P.q_len;
        __syncthreads();
        for (int i = tid; i < kGenHeads * D; i += blockDim.x) {
            const int hh = i / D, d = i - hh * D;
            const int h = h0 + hh;
            sq[hh * Dp + d] = h < P.H ? bf16_to_f32(P.q[(static_cast<int64_t>(g) * P.H + h) * D + d]) : 0.f;
        }
        if (tid < kGenHeads) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
        float acc[kGenMaxCols];
#pragma unroll
        for (int k = 0; k < kGenMaxCols; ++k) acc[k] = 0.f;

        for (int32_t t0 = seg.tok_begin; t0 < seg.tok_end; t0 += kGenTokens) {
            const int nt = min(kGenTokens, seg.tok_end - t0);
            __syncthreads();
            // stage this sub-tile's cache rows (bf16 -> fp32); missing rows read as zeros
            for (int i = tid; i < kGenTokens * (D / 8); i += blockDim.x) {
                const int tt = i / (D / 8), c8 = (i - tt * (D / 8)) * 8;
                float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (tt < nt) {
                    const int64_t row = resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks,
                                                    P.block_size, b, t0 + tt);
                    if (row >= 0) {
                        const uint4 u = *reinterpret_cast<const uint4*>(P.pool + row * D + c8);
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[2 * k] = __uint_as_float(w[k] << 16);
                            v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
                        }
                    } else if (c8 == 0) {
                        record_status(MLA_ERR_DEVICE_FAULT);
                    }
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) skv[tt * Dp + c8 + k] = v[k];
            }
            __syncthreads();
            // scores: thread -> (head hh, tokens tt, tt + 16)
            {
                const int hh = tid / 16, ta = tid % 16;
                const float* qr = sq + hh * Dp;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int tt = ta + 16 * r;
                    const float* kr = skv + tt * Dp;
                    float z = 0.f;
                    for (int d = 0; d < D; ++d) z = fmaf(qr[d], kr[d], z);
                    ss[hh * kGenTokens + tt] = tt < nt ? z * P.scale : -INFINITY;
                }
            }
            __syncthreads();
            // online softmax: one warp per two heads (16 lanes per head)
            {
                const int hh = tid / 16, lane16 = tid % 16;
                float* row = ss + hh * kGenTokens;
                float mx = fmaxf(row[lane16], row[lane16 + 16]);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const float m_old = s_m[hh];
                const float m_new = fmaxf(m_old, mx);
                float psum = 0.f;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float z = row[lane16 + 16 * r];
                    const float p = z == -INFINITY ? 0.f : __expf(z - m_new);
                    psum += p;
                    row[lane16 + 16 * r] = bf16_to_f32(f32_to_bf16(p));
                }
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
                __syncwarp();
                if (lane16 == 0) {
                    const float a = m_old == -INFINITY ? 0.f : __expf(m_old - m_new);
                    s_a[hh] = a;
                    s_l[hh] = s_l[hh] * a + psum;
                    s_m[hh] = m_new;
                }
            }
            __syncthreads();
            // value sum: thread -> (head hl, columns cl + 16 k)
            {
                const float a = s_a[hl];
                const float* pr = ss + hl * kGenTokens;
#pragma unroll
                for (int k = 0; k < kGenMaxCols; ++k) {
                    if (k < ncol) {
                        const int c = cl + 16 * k;
                        float v = acc[k] * a;
                        if (c < P.dc)
                            for (int tt = 0; tt < nt; ++tt) v = fmaf(pr[tt], skv[tt * Dp + c], v);
                        acc[k] = v;
                    }
                }
            }
        }
        __syncthreads();
        const int h = h0 + hl;
        if (h < P.H) {
            const float l = s_l[hl];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            float* dst = P.o_part + (static_cast<int64_t>(seg.slot) * P.H + h) * P.dc;
#pragma unroll
            for (int k = 0; k < kGenMaxCols; ++k) {
                const int c = cl + 16 * k;
                if (k < ncol && c < P.dc) dst[c] = acc[k] * inv;
            }
            if (cl == 0)
                P.lse_part[static_cast<int64_t>(seg.slot) * P.H + h] = l > 0.f ? s_m[hl] + __logf(l) : -INFINITY;
        }
    }
}

}  // namespace mla
