// Split-KV schedule, computed on the device from the device-resident
// context lengths (so a decode step needs no host synchronisation).
//
// A "group" is one new token of one sequence: g = b * q_len + s. Group g
// sees vis(g) = L_b - q_len + s + 1 cached tokens (the causal rule for
// several new tokens), i.e. ceil(vis / tile) tiles. All groups' tiles are
// laid end to end (W tiles in total) and cut into P contiguous, non-empty
// ranges, one per worker: worker p owns tiles [floor(W p / P),
// floor(W (p+1) / P)). A worker emits one partial (o, lse) per group it
// touches; group g's partials are the consecutive slots
// part_offsets[g] .. part_offsets[g+1]-1, ordered by worker.
#pragma once

#include "common.cuh"

namespace mla {

struct PlanHeader {
    int32_t total_tiles;  // W
    int32_t workers;      // P (<= requested workers, <= W; 0 when W == 0)
    int32_t n_groups;     // G
    int32_t n_parts;      // part_offsets[G]
};

__host__ __device__ __forceinline__ int32_t worker_begin(int32_t p, int32_t W, int32_t P) {
    return static_cast<int32_t>((static_cast<int64_t>(W) * p) / P);
}

// The worker whose range holds tile t (largest p with worker_begin(p) <= t).
__host__ __device__ __forceinline__ int32_t worker_of_tile(int32_t t, int32_t W, int32_t P) {
    return static_cast<int32_t>(((static_cast<int64_t>(t) + 1) * P - 1) / W);
}

__device__ __forceinline__ int32_t group_tiles(const int32_t* __restrict__ context_lens, int32_t q_len,
                                               int32_t g, int32_t tile) {
    const int32_t b = g / q_len, s = g - b * q_len;
    const int32_t vis = __ldg(context_lens + b) - q_len + s + 1;
    return vis > 0 ? (vis + tile - 1) / tile : 0;
}

__device__ __forceinline__ int32_t group_visible(const int32_t* __restrict__ context_lens, int32_t q_len,
                                                 int32_t g) {
    const int32_t b = g / q_len, s = g - b * q_len;
    const int32_t vis = __ldg(context_lens + b) - q_len + s + 1;
    return vis > 0 ? vis : 0;
}

// Largest g with tile_prefix[g] <= t (the non-empty group owning tile t).
__device__ __forceinline__ int32_t group_of_tile(const int32_t* __restrict__ tile_prefix, int32_t G, int32_t t) {
    int32_t lo = 0, hi = G - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Exclusive block-wide scan of one value per thread (blockDim.x == 1024).
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_tot, int32_t* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int32_t w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive over warps
        if (lane == 31) *total = w;
    }
    __syncthreads();
    const int32_t base = wid ? warp_tot[wid - 1] : 0;
    const int32_t r = base + x - v;
    __syncthreads();
    return r;
}

// <<<1, 1024>>>. tile_prefix and part_offsets have G + 1 entries.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ context_lens, int32_t batch,
                                                    int32_t q_len, int32_t tile, int32_t max_workers,
                                                    PlanHeader* __restrict__ hdr,
                                                    int32_t* __restrict__ tile_prefix,
                                                    int32_t* __restrict__ part_offsets) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t chunk_total;
    const int32_t G = batch * q_len;
    int32_t carry = 0;
    for (int32_t base = 0; base < G; base += 1024) {
        const int32_t g = base + threadIdx.x;
        const int32_t n = g < G ? group_tiles(context_lens, q_len, g, tile) : 0;
        const int32_t ex = block_exclusive_scan(n, warp_tot, &chunk_total);
        if (g < G) tile_prefix[g] = carry + ex;
        carry += chunk_total;
        __syncthreads();
    }
    const int32_t W = carry;
    const int32_t P = W > 0 ? min(max_workers, W) : 0;
    if (threadIdx.x == 0) tile_prefix[G] = W;
    __syncthreads();
    carry = 0;
    for (int32_t base = 0; base < G; base += 1024) {
        const int32_t g = base + threadIdx.x;
        int32_t n = 0;
        if (g < G) {
            const int32_t t0 = tile_prefix[g], t1 = tile_prefix[g + 1];
            if (t1 > t0) n = worker_of_tile(t1 - 1, W, P) - worker_of_tile(t0, W, P) + 1;
        }
        const int32_t ex = block_exclusive_scan(n, warp_tot, &chunk_total);
        if (g < G) part_offsets[g] = carry + ex;
        carry += chunk_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        part_offsets[G] = carry;
        hdr->total_tiles = W;
        hdr->workers = P;
        hdr->n_groups = G;
        hdr->n_parts = carry;
    }
}

// One contiguous run of a worker's tiles inside a single group.
struct Segment {
    int32_t group;
    int32_t tok_begin, tok_end;  // token range [tok_begin, tok_end) of the group's visible tokens
    int32_t slot;                // partial slot
};

// Iterates the segments of worker p. Usage:
//   SegmentIter it(...); Segment s; while (it.next(s)) { ... }
struct SegmentIter {
    const int32_t* tile_prefix;
    const int32_t* part_offsets;
    const int32_t* context_lens;
    int32_t G, q_len, tile, W, P, p;
    int32_t t, t_end;

    __device__ SegmentIter(const PlanHeader* hdr, const int32_t* tp, const int32_t* po, const int32_t* cl,
                           int32_t q_len_, int32_t tile_, int32_t worker)
        : tile_prefix(tp), part_offsets(po), context_lens(cl), q_len(q_len_), tile(tile_), p(worker) {
        G = hdr->n_groups;
        W = hdr->total_tiles;
        P = hdr->workers;
        if (p < P) {
            t = worker_begin(p, W, P);
            t_end = worker_begin(p + 1, W, P);
        } else {
            t = t_end = 0;
        }
    }

    __device__ bool next(Segment& s) {
        if (t >= t_end) return false;
        const int32_t g = group_of_tile(tile_prefix, G, t);
        const int32_t g0 = tile_prefix[g], g1 = tile_prefix[g + 1];
        const int32_t hi = min(t_end, g1);
        const int32_t vis = group_visible(context_lens, q_len, g);
        s.group = g;
        s.tok_begin = (t - g0) * tile;
        s.tok_end = min((hi - g0) * tile, vis);
        s.slot = part_offsets[g] + (p - worker_of_tile(g0, W, P));
        t = hi;
        return true;
    }
};

}  // namespace mla
