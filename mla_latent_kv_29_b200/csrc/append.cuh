// Cache append: the joint down-projection kv = x . W_kva
// (kv_a_proj_with_mqa, "MLA架构：低秩注意力机制优化LLM显存与计算效率" 2.2),
// then RMSNorm on the c_kv part (kv_a_layernorm), rotate-half RoPE on the
// k_pe part ("一次讲透MHA、GQA、MQA、MLA", "MLA的实现", RoPE module) and the
// write of the bf16 row into its paged slot -- RoPE fused with the cache
// update as section 4.2 of the first page suggests.
//
// Two launches: a split-K GEMM writing fp32 partial sums, then one CTA per
// token that reduces the splits and runs the normalise / rotate / scatter
// epilogue (the RMSNorm needs the whole 512-wide row). The epilogue writes a
// bf16 row, or (fp8 set) the row of the FP8 cache (fp8.cuh): c rounded to
// bf16 first, its e4m3 codes under the per-token power-of-two scale, and k_pe
// as f16.
#pragma once

#include "common.cuh"
#include "fp8.cuh"

namespace mla {

constexpr int kApTileT = 64, kApTileN = 64, kApTileK = 32;

// grid (ceil(N / 64), ceil(T / 64), splits); block 256.
// part[split][T][N] = sum over this split's K range of x[t][k] * w[k][n].
__global__ void __launch_bounds__(256) append_gemm_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, float* __restrict__ part,
    int32_t T, int32_t K, int32_t N, int32_t k_per_split) {
    pdl_wait();
    pdl_trigger();
    __shared__ float xs[kApTileK][kApTileT + 4];  // k-major so the inner loop reads rows
    __shared__ float ws[kApTileK][kApTileN + 4];
    const int n0 = blockIdx.x * kApTileN, t0 = blockIdx.y * kApTileT;
    const int k_begin = blockIdx.z * k_per_split;
    const int k_end = min(K, k_begin + k_per_split);
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = k_begin; k0 < k_end; k0 += kApTileK) {
        for (int i = threadIdx.x; i < kApTileT * kApTileK; i += 256) {
            const int tt = i / kApTileK, kk = i % kApTileK;
            const int t = t0 + tt, k = k0 + kk;
            xs[kk][tt] = (t < T && k < k_end) ? bf16_to_f32(x[static_cast<int64_t>(t) * K + k]) : 0.f;
        }
        for (int i = threadIdx.x; i < kApTileK * kApTileN; i += 256) {
            const int kk = i / kApTileN, nn = i % kApTileN;
            const int k = k0 + kk, n = n0 + nn;
            ws[kk][nn] = (k < k_end && n < N) ? bf16_to_f32(w[static_cast<int64_t>(k) * N + n]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kApTileK; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* dst = part + static_cast<int64_t>(blockIdx.z) * T * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) dst[static_cast<int64_t>(t) * N + n] = acc[i][j];
        }
    }
}

struct AppendEpilogueParams {
    const float* part;  // [splits][T][N]
    const uint16_t* gamma;  // [dc] or null
    const int32_t* seq_ids;
    const int32_t* positions;
    const int32_t* block_table;
    uint16_t* pool;        // bf16 rows (fp8 = 0)
    uint8_t* pool8;        // FP8 blocks (fp8 = 1)
    fp8::Layout layout8;   // row / scale offsets of the FP8 blocks
    int32_t fp8;
    int64_t num_blocks;
    int32_t splits, T, dc, dr, num_seqs, max_blocks_per_seq, block_size;
    float eps;
    double rope_base;
};

// RoPE angle of pair i at position pos: pos * base^(-2i/dr), formed in double and
// reduced to [-pi, pi] with a two-term 2*pi so the float sine/cosine stay on
// their short-argument path.
__device__ __forceinline__ void rope_sincos(int32_t pos, int i, int dr, double base, float* s, float* c) {
    const double inv_freq = exp2(-2.0 * i / static_cast<double>(dr) * log2(base));
    const double angle = static_cast<double>(pos) * inv_freq;
    const double k = rint(angle * 0.15915494309189535);  // 1 / (2 pi)
    const double reduced = fma(-k, 2.4492935982947064e-16, fma(-k, 6.283185307179586, angle));
    sincosf(static_cast<float>(reduced), s, c);
}

// grid (T); block 256; dynamic smem (dc + dr) floats.
__global__ void __launch_bounds__(256) append_epilogue_kernel(AppendEpilogueParams P) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float kv[];
    __shared__ float red[32];
    const int t = blockIdx.x;
    const int N = P.dc + P.dr;
    const int64_t split_stride = static_cast<int64_t>(P.T) * N;
    // kv[n] = sum over splits; each thread owns columns threadIdx.x + 256 i (i < 3 for
    // N = 576) and requests eight splits of all its columns before summing them, so
    // the loads of a thread are independent and few memory round trips are exposed.
    constexpr int kCols = 4;  // N <= 1024
    constexpr int kBatch = 8;
    float acc[kCols] = {0.f, 0.f, 0.f, 0.f};
    const float* src = P.part + static_cast<int64_t>(t) * N + threadIdx.x;
    for (int k0 = 0; k0 < P.splits; k0 += kBatch) {
        float v[kBatch][kCols];
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
#pragma unroll
            for (int i = 0; i < kCols; ++i) {
                const int n = static_cast<int>(threadIdx.x) + 256 * i;
                v[u][i] = (k0 + u < P.splits && n < N) ? __ldg(src + (k0 + u) * split_stride + 256 * i) : 0.f;
            }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
#pragma unroll
            for (int i = 0; i < kCols; ++i) acc[i] += v[u][i];
    }
#pragma unroll
    for (int i = 0; i < kCols; ++i) {
        const int n = static_cast<int>(threadIdx.x) + 256 * i;
        if (n < N) kv[n] = acc[i];
    }
    __syncthreads();
    // RMSNorm over the latent part
    float ss = 0.f;
    for (int n = threadIdx.x; n < P.dc; n += blockDim.x) ss = fmaf(kv[n], kv[n], ss);
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        v = warp_sum(v);
        if (threadIdx.x == 0) red[0] = rsqrtf(v / static_cast<float>(P.dc) + P.eps);
    }
    __syncthreads();
    const float r = red[0];
    const int32_t b = P.seq_ids[t], pos = P.positions[t];
    const int64_t row = resolve_row(P.block_table, P.num_seqs, P.max_blocks_per_seq, P.num_blocks, P.block_size, b, pos);
    if (row < 0) {
        if (threadIdx.x == 0) record_status(MLA_ERR_DEVICE_FAULT);
        return;
    }
    const int half = P.dr / 2;
    if (P.fp8) {
        // c as the bf16 cache would hold it, kept in kv[] for the encode pass
        float amax = 0.f;
        for (int n = threadIdx.x; n < P.dc; n += blockDim.x) {
            float c = kv[n] * r;
            if (P.gamma) c *= bf16_to_f32(P.gamma[n]);
            c = bf16_to_f32(f32_to_bf16(c));
            kv[n] = c;
            amax = fmaxf(amax, fabsf(c));
        }
        amax = warp_max(amax);
        __syncthreads();  // every thread has read red[0]
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
        amax = 0.f;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
        const int e = fp8::scale_exp(amax);
        const float inv = fp8::pow2(-e);
        uint8_t* d8 = P.pool8 + P.layout8.row_off(row);
        uint16_t* codes = reinterpret_cast<uint16_t*>(d8);
        for (int n2 = threadIdx.x; n2 < P.dc / 2; n2 += blockDim.x)
            codes[n2] = fp8::e4m3x2(kv[2 * n2] * inv, kv[2 * n2 + 1] * inv);
        uint16_t* pe = reinterpret_cast<uint16_t*>(d8 + P.dc);
        for (int i = threadIdx.x; i < half; i += blockDim.x) {
            float s, c;
            rope_sincos(pos, i, P.dr, P.rope_base, &s, &c);
            const float x1 = kv[P.dc + i], x2 = kv[P.dc + i + half];
            pe[i] = fp8::f16_bits(x1 * c - x2 * s);
            pe[i + half] = fp8::f16_bits(x2 * c + x1 * s);
        }
        if (threadIdx.x == 0) *reinterpret_cast<float*>(P.pool8 + P.layout8.scale_off(row)) = fp8::pow2(e);
        return;
    }
    uint16_t* dst = P.pool + row * N;
    for (int n = threadIdx.x; n < P.dc; n += blockDim.x) {
        float c = kv[n] * r;
        if (P.gamma) c *= bf16_to_f32(P.gamma[n]);
        dst[n] = f32_to_bf16(c);
    }
    // rotate-half RoPE: pair (i, i + dr/2) rotated by pos * base^(-2i/dr)
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        float s, c;
        rope_sincos(pos, i, P.dr, P.rope_base, &s, &c);
        const float x1 = kv[P.dc + i], x2 = kv[P.dc + i + half];
        dst[P.dc + i] = f32_to_bf16(x1 * c - x2 * s);
        dst[P.dc + i + half] = f32_to_bf16(x2 * c + x1 * s);
    }
}

// Test hook: rows of (seq, pos) through the shared resolver.
__global__ void resolve_slots_kernel(const int32_t* __restrict__ block_table, int32_t num_seqs, int32_t max_blocks_per_seq,
                                     int64_t num_blocks, int32_t block_size, const int32_t* __restrict__ seq_ids,
                                     const int32_t* __restrict__ positions, int32_t n, int64_t* __restrict__ rows) {
    pdl_wait();
    pdl_trigger();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) rows[i] = resolve_row(block_table, num_seqs, max_blocks_per_seq, num_blocks, block_size, seq_ids[i], positions[i]);
}

}  // namespace mla
