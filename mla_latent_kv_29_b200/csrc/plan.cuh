// Split-KV schedule, computed on the device from the device-resident
// context lengths (so a decode step needs no host synchronisation).
//
// A "group" is one new token of one sequence: g = b * q_len + s. Group g
// sees vis(g) = L_b - q_len + s + 1 cached tokens (the causal rule for
// several new tokens), i.e. n_g = ceil(vis / tile) tiles. Every segment a
// worker runs costs a fixed start-up (query load, pipeline fill, partial
// write-out) on top of its tiles, so the schedule is cut in "units": each
// group contributes kSegUnits units for that cost followed by one unit per
// tile. Group g starts at unit V0(g) = tile_prefix[g] + kSegUnits * g; its
// tile k sits at unit V0(g) + kSegUnits + k. The W' = V0(G) units are cut
// into P contiguous ranges, worker p owning [floor(W' p / P), floor(W' (p+1) / P)).
// A worker emits one partial (o, lse) per group whose tiles it touches;
// group g's partials are the consecutive slots part_offsets[g] ..
// part_offsets[g+1]-1, ordered by worker. worker_group[p] is the group whose
// units hold the start of worker p's range.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int32_t kSegUnits = 1;  // schedule units charged per segment (about one tile of time)

struct PlanHeader {
    int32_t total_units;  // W' (0 when no group has a visible token)
    int32_t workers;      // P (<= requested workers, <= W'; 0 when W' == 0)
    int32_t n_groups;     // G
    int32_t n_parts;      // part_offsets[G]
};

__host__ __device__ __forceinline__ int32_t worker_begin(int32_t p, int32_t W, int32_t P) {
    return static_cast<int32_t>((static_cast<int64_t>(W) * p) / P);
}

// The worker whose range holds unit v (largest p with worker_begin(p) <= v).
__host__ __device__ __forceinline__ int32_t worker_of_unit(int32_t v, int32_t W, int32_t P) {
    return static_cast<int32_t>(((static_cast<int64_t>(v) + 1) * P - 1) / W);
}

__device__ __forceinline__ int32_t group_units_start(const int32_t* __restrict__ tile_prefix, int32_t g) {
    return tile_prefix[g] + kSegUnits * g;
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

// Largest g in [0, G) with V0(g) <= v (the group whose units hold unit v).
__device__ __forceinline__ int32_t group_of_unit(const int32_t* __restrict__ tile_prefix, int32_t G, int32_t v) {
    int32_t lo = 0, hi = G - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (group_units_start(tile_prefix, mid) <= v) lo = mid; else hi = mid - 1;
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

// <<<1, 1024, smem>>>. tile_prefix and part_offsets have G + 1 entries,
// worker_group max_workers entries. With smem = 4 (G + 1) bytes of dynamic
// shared memory (prefix_in_smem) the later passes read the prefix, and the
// binary searches of group_of_unit run, in shared memory instead of chains of
// dependent global loads.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ context_lens, int32_t batch,
                                                    int32_t q_len, int32_t tile, int32_t max_workers,
                                                    PlanHeader* __restrict__ hdr,
                                                    int32_t* __restrict__ tile_prefix,
                                                    int32_t* __restrict__ part_offsets,
                                                    int32_t* __restrict__ worker_group, int32_t prefix_in_smem) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t chunk_total;
    extern __shared__ int32_t s_prefix[];
    int32_t* tp = prefix_in_smem ? s_prefix : tile_prefix;  // where the later passes read the prefix
    const int32_t G = batch * q_len;
    int32_t carry = 0;
    for (int32_t base = 0; base < G; base += 1024) {
        const int32_t g = base + threadIdx.x;
        const int32_t n = g < G ? group_tiles(context_lens, q_len, g, tile) : 0;
        const int32_t ex = block_exclusive_scan(n, warp_tot, &chunk_total);
        if (g < G) {
            tile_prefix[g] = carry + ex;
            if (prefix_in_smem) s_prefix[g] = carry + ex;
        }
        carry += chunk_total;
        __syncthreads();
    }
    const int32_t W = carry > 0 ? carry + kSegUnits * G : 0;
    const int32_t P = W > 0 ? min(max_workers, W) : 0;
    if (threadIdx.x == 0) {
        tile_prefix[G] = carry;
        if (prefix_in_smem) s_prefix[G] = carry;
    }
    __syncthreads();
    carry = 0;
    for (int32_t base = 0; base < G; base += 1024) {
        const int32_t g = base + threadIdx.x;
        int32_t n = 0;
        if (g < G) {
            const int32_t t0 = tp[g], t1 = tp[g + 1];
            if (t1 > t0) {
                const int32_t v0 = t0 + kSegUnits * (g + 1);  // unit of the group's first tile
                n = worker_of_unit(v0 + (t1 - t0) - 1, W, P) - worker_of_unit(v0, W, P) + 1;
            }
        }
        const int32_t ex = block_exclusive_scan(n, warp_tot, &chunk_total);
        if (g < G) part_offsets[g] = carry + ex;
        carry += chunk_total;
        __syncthreads();
    }
    for (int32_t p = threadIdx.x; p < P; p += 1024)
        worker_group[p] = group_of_unit(tp, G, worker_begin(p, W, P));
    if (threadIdx.x == 0) {
        part_offsets[G] = carry;
        hdr->total_units = W;
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
    int32_t g, v, v_end;  // next group to look at; this worker's unit range [v, v_end)

    __device__ SegmentIter(const PlanHeader* hdr, const int32_t* worker_group, const int32_t* tp, const int32_t* po,
                           const int32_t* cl, int32_t q_len_, int32_t tile_, int32_t worker)
        : tile_prefix(tp), part_offsets(po), context_lens(cl), q_len(q_len_), tile(tile_), p(worker) {
        G = hdr->n_groups;
        W = hdr->total_units;
        P = hdr->workers;
        if (p < P) {
            v = worker_begin(p, W, P);
            v_end = worker_begin(p + 1, W, P);
            g = worker_group[p];
        } else {
            v = v_end = 0;
            g = G;
        }
    }

    __device__ bool next(Segment& s) {
        while (g < G) {
            const int32_t t0 = tile_prefix[g], t1 = tile_prefix[g + 1];
            const int32_t u = t0 + kSegUnits * (g + 1);  // unit of the group's first tile
            if (u - kSegUnits >= v_end) break;
            const int32_t k0 = max(0, v - u), k1 = min(t1 - t0, v_end - u);
            const int32_t gg = g++;
            if (k1 <= k0) continue;
            s.group = gg;
            s.tok_begin = k0 * tile;
            s.tok_end = min(k1 * tile, group_visible(context_lens, q_len, gg));
            s.slot = part_offsets[gg] + (p - worker_of_unit(u, W, P));
            return true;
        }
        g = G;
        return false;
    }
};

}  // namespace mla
