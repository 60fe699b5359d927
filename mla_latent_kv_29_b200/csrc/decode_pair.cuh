// Split-KV absorbed MLA attention on the sm_100a tensor cores (DeepSeek-V3
// dims: 128 heads, latent 512, RoPE 64).
//
// Per new token g and split segment [tok_begin, tok_end) of its visible
// tokens: S = scale * [q_lat ; q_pe] . [c ; k_pe]^T over all 128 heads at once
// (the absorbed score of "一次讲透MHA、GQA、MQA、MLA", section "MLA的实现"; all
// heads share the latent tile, so it is a dense [128 x 576] . [576 x tokens]
// contraction), online softmax, O += P . c (the [128 x tokens] .
// [tokens x 512] value contraction), then the normalised partial (O / l,
// lse) of the segment.
//
// Work split. One worker is a cluster of two CTAs (a pair). Tensor-core MMAs
// are issued by the pair's leader with cta_group::2 and M = 128 heads: CTA r
// holds heads 64r..64r+63 of every operand A (queries, softmax weights) and
// of every accumulator, folded over all 128 TMEM lanes (columns [0, N/2) of
// the result in lanes 0-63, [N/2, N) in lanes 64-127), and supplies half of
// every operand B:
//   S MMA  (M 128, N 128 tokens, K 576): CTA r supplies the 64 tokens of its
//          page of the 128-token tile (all 576 values per token);
//   PV MMA (M 128, N 256 latent columns, K 128 tokens), twice per tile:
//          CTA r supplies latent columns 256r + 128n .. +127 for all tokens.
// The tile's latent values therefore reach each CTA twice (once as keys,
// once as values), so shared-memory fills are ~1.9x the HBM bytes, while
// HBM reads stay ~1x because the second read of a page hits L2 (each CTA
// also asks L2 for its page of the next tile ahead of the key loads).
//
// Warp roles per CTA (320 threads): one thread of warp 0 streams the queries
// and the key stages (column blocks 0-2, 3-4, 5-6 and 7-8 of the CTA's page,
// one TMA operation each) into a one-tile key ring; warp 2 streams the value
// stages (32 tokens x 256 columns, 16 KB) into a four-stage value ring that
// holds a whole tile (one thread issues, the warp zeroes the tail rows of
// partial stages); warp 1 allocates tensor memory (both CTAs). In the leader,
// four threads issue the MMAs, each its own independent stream: lanes 0 of
// warps 1 and 3 the score MMAs of every tile (column blocks 0-4 and 5-8,
// into two half-accumulators that the softmax adds), lanes 0 of warps 8 and 9
// the value MMAs (latent columns 0-255 and 256-511 of the pair's O). One
// thread cannot issue the M 128 x N 128 score instructions as fast as the
// tensor cores run them, and a thread stalls at each wait for its operands,
// so independent streams keep the tensor pipe fed while any one of them waits.
// Warps 4-7 (thread t = TMEM lane t) run the softmax, rescale O when the
// running max grows by more than 2^8, write P to shared memory (one buffer,
// rewritten once the value MMAs of the previous tile are done) and, at the
// end of a segment, normalise O and write the partial.
// Every mbarrier wait is bounded (see ptx::mbar_wait; the limit is a kernel
// parameter so that a test can shorten it): on expiry the kernel records
// MLA_ERR_DEVICE_TIMEOUT and every role drains to the common exit. With the
// test hook `starve` the load warps issue nothing at all, so no copy or
// tensor-core operation is in flight when the consumers' waits run out.
//
// FP8 cache (pair_decode_f8_kernel; the format is in fp8.cuh). The same
// pipeline with f16 operands: the absorbed queries arrive as f16, the softmax
// writes P as f16, and every cache box is expanded in place. The load warps
// copy each [rows x 64] box of e4m3 codes (64 bytes a row, unswizzled) into
// the upper half of the shared-memory box that will hold its f16 values, and
// the token scales into the lower half of the stage's first box; two more
// warps (384 threads) turn them into exactly the 128B-swizzled f16 boxes the
// bf16 path loads directly (warp 10 the key stages, warp 11 the value stages,
// zeroing value rows past the visible range), then signal the stage full to
// the leader. Each warp reads a box's codes and scales into registers before
// any lane writes it. The f16 RoPE key box is copied as it is. HBM bytes per
// token: 644 instead of 1152.
#pragma once

#include "common.cuh"
#include "plan.cuh"
#include "sm100.cuh"
#include "fp8.cuh"

namespace mla {
namespace pair {

constexpr int kH = 128, kDc = 512, kDr = 64, kD = kDc + kDr;
constexpr int kTile = 128;       // tokens per pair iteration
constexpr int kBox = 8192;       // one [64 rows x 64 bf16] 128B-swizzled box
constexpr int kQBoxes = kD / 64; // 9
// Key ring: one tile = the CTA's page as 9 [64 x 64] boxes in column-block
// order, filled as 4 stages (blocks 0-2, 3-4, 5-6, 7-8). The score MMAs of a
// tile are split by column blocks between two issuing threads: "lo" takes
// blocks 0-4 (stages 0, 1) into one accumulator, "hi" blocks 5-8 (stages 2,
// 3) into another, and the softmax adds the two.
constexpr int kKStages = 4;
__host__ __device__ constexpr int kstage_first_block(int s) { return s == 0 ? 0 : 1 + 2 * s; }
__host__ __device__ constexpr int kstage_blocks(int s) { return s == 0 ? 3 : 2; }
constexpr int kKTile = kQBoxes * kBox;  // 72 KB
constexpr int kVStage = 2 * kBox;    // value stage: 32 tokens x 256 latent columns (4 x 4 KB)
constexpr int kVPerTile = 4;         // 4 value stages per tile
constexpr int kVStages = 4;          // value ring: four stages (a whole tile)
constexpr int kThreads = 320;  // 10 warps; the softmax warps 4-7 own TMEM lanes 0-127
constexpr int kF8Threads = 384;  // FP8 cache: + warp 10 (key expansion) and warp 11 (value expansion)
constexpr int kF8Row = kDc + 2 * kDr;  // 640 bytes: 512 e4m3 codes, then the f16 RoPE key
constexpr int kF8KSrc = kBox / 2;      // a key box's 64 rows of 64 codes sit in its upper 4 KB
constexpr int kF8VSrc = kBox / 4;      // a value box's 32 rows of 64 codes sit in its upper 2 KB
constexpr int kTmemCols = 512;
constexpr int kTmS = 0;          // two S buffers (tile parity), each lo and hi halves of 64 columns
constexpr int kTmO = 256;        // O: 256 columns (after the two S buffers of 128)

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBoxes * kBox;
constexpr int kOffV = kOffK + kKTile;
constexpr int kOffP = kOffV + kVStages * kVStage;
constexpr int kOffBar = kOffP + 2 * kBox;  // one P buffer of 2 boxes

enum Bar {
    B_QFULL = 0, B_QEMPTY, B_SFULL0, B_SFULL1, B_SEMPTY0, B_SEMPTY1, B_PFULL0, B_PFULL1, B_PVDONE0, B_PVDONE1,
    B_OEMPTY, B_PATCH, B_XCHG,
    B_KFULL0, B_KEMPTY0 = B_KFULL0 + kKStages, B_VFULL0 = B_KEMPTY0 + kKStages, B_VEMPTY0 = B_VFULL0 + kVStages,
    B_KRAW0 = B_VEMPTY0 + kVStages, B_VRAW0 = B_KRAW0 + kKStages,  // FP8: codes landed (this CTA)
    B_COUNT = B_VRAW0 + kVStages
};
constexpr int kOffRed = kOffBar + 8 * 64;          // exchange buffer [2][128] floats
constexpr int kOffMisc = kOffRed + 2 * 128 * 4;    // abort flag, TMEM base
constexpr int kSmemBytes = kOffMisc + 64 + 1024;   // + slack to align the base to 1 KB
static_assert(B_COUNT <= 64, "barrier area");
static_assert(kTmS + 2 * 128 <= kTmO && kTmO + 256 <= kTmemCols, "tensor memory map: S buffers, then O");
static_assert(kstage_first_block(kKStages - 1) + kstage_blocks(kKStages - 1) == kQBoxes, "key stages cover a page");

struct Params {
    const PlanHeader* hdr;
    const int32_t* worker_group;
    const int32_t* tile_prefix;
    const int32_t* part_offsets;
    const int32_t* context_lens;
    const int32_t* block_table;
    const uint8_t* pool;  // the cache rows (for the L2 prefetch of upcoming pages)
    uint16_t* o_part;  // [n_parts, 128, 512] bf16 (normalised partial outputs)
    float* lse_part;  // [n_parts, 128]
    int64_t num_blocks;
    int32_t batch, max_blocks_per_seq, block_size, q_len;
    float scale_log2;  // softmax_scale * log2(e)
    uint64_t wait_ns;  // limit of every bounded wait (ptx::kWaitLimitNs unless a test shortens it)
    int32_t starve;    // test hook: the load warps issue nothing, so every consumer wait runs out
    int64_t f8_block_bytes;  // FP8 cache: bytes of one cache block (rows, then scales)
};

struct Ctx {
    uint8_t* smem;
    uint32_t sbase;
    uint32_t rank;
    uint32_t pair;
    uint32_t tmem;
    volatile int* abort;
    uint64_t wait_ns;  // limit of every mbarrier wait
    __device__ uint32_t bar(int i) const { return sbase + kOffBar + 8 * i; }
    __device__ uint32_t leader_bar(int i) const { return ptx::mapa(bar(i), 0); }
};

__device__ __forceinline__ int tiles_of(const Segment& s) { return (s.tok_end - s.tok_begin + kTile - 1) / kTile; }

// ------------------------------------------------------------------ producer
template <int N>
__device__ __forceinline__ void ring_next(uint32_t& stage, uint32_t& phase) {
    if (++stage == N) { stage = 0; phase ^= 1; }
}

// Starts pulling this CTA's 64-token page of tile j of `seg` (73,728
// contiguous bytes: the 64 rows lie in one pool block because block_size is a
// multiple of 64; FP8: 40,960 bytes of rows and the page's 256 bytes of
// scales) from HBM into L2, so that its key loads a tile later hit L2.
template <bool kF8>
__device__ __forceinline__ void prefetch_page(const Params& P, const Ctx& c, const Segment& seg, int j) {
    const int32_t th = seg.tok_begin + j * kTile + 64 * static_cast<int32_t>(c.rank);
    if (th >= seg.tok_end) return;
    const int64_t row = resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size,
                                    seg.group / P.q_len, th);
    if (row < 0) return;
    if (kF8) {
        const int64_t blk = row / P.block_size, slot = row % P.block_size;
        const uint8_t* base = P.pool + blk * P.f8_block_bytes;
        ptx::prefetch_l2(base + slot * kF8Row, 64 * kF8Row);
        ptx::prefetch_l2(base + static_cast<int64_t>(P.block_size) * kF8Row + 4 * slot, 64 * 4);
    } else {
        ptx::prefetch_l2(P.pool + row * (kD * 2), 64 * kD * 2);
    }
}

// Queries and key stages; one thread (lane 0 of warp 0). tm_q, tm_k3 and
// tm_k2 are 3-D maps {64 columns, rows, 9 column blocks} with boxes
// {64, 64, 9}, {64, 64, 3} and {64, 64, 2}: one TMA operation fills the whole
// query block or a key stage. Before the loads of tile j it asks L2 for the
// page of the tile after it (in this segment or the next).
__device__ void key_producer(const Params& P, const CUtensorMap* tm_q, const CUtensorMap* tm_k3,
                             const CUtensorMap* tm_k2, const Ctx& c) {
    uint32_t phase = 0;  // parity of the pair's running tile count
    int seg_i = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    {
        SegmentIter peek = it;
        if (peek.next(seg)) prefetch_page<false>(P, c, seg, 0);
    }
    while (it.next(seg)) {
        const int32_t g = seg.group, b = g / P.q_len;
        if (seg_i > 0 && !ptx::mbar_wait(c.bar(B_QEMPTY), (seg_i - 1) & 1, c.abort, c.wait_ns)) return;
        {
            const uint32_t full = c.leader_bar(B_QFULL);
            ptx::mbar_arrive_expect_tx_cluster(full, kQBoxes * kBox);
            ptx::tma_load_3d_pair(c.sbase + kOffQ, tm_q, 0, g * kH + 64 * c.rank, 0, full);
        }
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            // this CTA's 64-token page of tile j, all 576 values
            const int32_t t0 = seg.tok_begin + j * kTile;
            int32_t th = t0 + 64 * static_cast<int32_t>(c.rank);
            if (th >= seg.tok_end) th = t0;  // no visible token in this half: any valid page (masked)
            int64_t row = resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size,
                                      b, th);
            if (row < 0) {
                record_status(MLA_ERR_DEVICE_FAULT);
                row = 0;
            }
            if (j + 1 < n_tiles) {
                prefetch_page<false>(P, c, seg, j + 1);
            } else {
                SegmentIter peek = it;
                Segment nx;
                if (peek.next(nx)) prefetch_page<false>(P, c, nx, 0);
            }
            for (int ks = 0; ks < kKStages; ++ks) {
                if (!ptx::mbar_wait(c.bar(B_KEMPTY0 + ks), phase ^ 1, c.abort, c.wait_ns)) return;
                const uint32_t full = c.leader_bar(B_KFULL0 + ks);
                const int blk = kstage_first_block(ks);
                ptx::mbar_arrive_expect_tx_cluster(full, kstage_blocks(ks) * kBox);
                ptx::tma_load_3d_pair(c.sbase + kOffK + blk * kBox, ks == 0 ? tm_k3 : tm_k2, 0,
                                      static_cast<int32_t>(row), blk, full);
            }
            phase ^= 1;
        }
        ++seg_i;
    }
    // Tail: wait until the MMA has released every key stage and the last query
    // block, so that no asynchronous arrival (a multicast tcgen05.commit) can
    // reach this CTA's shared memory after it exits -- it would land in the
    // barriers of whatever CTA runs here next.
    for (int ks = 0; ks < kKStages; ++ks)
        if (!ptx::mbar_wait(c.bar(B_KEMPTY0 + ks), phase ^ 1, c.abort, c.wait_ns)) return;
    if (seg_i > 0) ptx::mbar_wait(c.bar(B_QEMPTY), (seg_i - 1) & 1, c.abort, c.wait_ns);
}

// Value stages; warp 2 (lane 0 issues and waits, the whole warp zeroes the
// tail rows of a partial stage). Stage q of a tile holds tokens 32q..32q+31
// and this CTA's latent columns 256r..256r+255 as four 4 KB boxes: box (n, h)
// = columns 256r + 128n + 64h at offset (2n + h) * 4 KB. tm_v is a 3-D map
// {64 columns, rows, 9 column blocks} with box {64, 32, 4}: one TMA operation
// fills a stage. Stages that hold no visible token are skipped here and by
// the value-MMA issuer alike (their softmax weights are all zero).
__device__ void value_producer(const Params& P, const CUtensorMap* tm_v, const Ctx& c) {
    const uint32_t lane = ptx::lane_id();
    uint32_t stage = 0, phase = 0, patch_phase = 0;
    // a wait by lane 0, its outcome shared so that the warp stays converged
    auto wait0 = [&](uint32_t bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0) ok = ptx::mbar_wait(bar, parity, c.abort, c.wait_ns) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        const int32_t b = seg.group / P.q_len;
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const int32_t tv = seg.tok_begin + j * kTile;
            for (int q = 0; q < kVPerTile; ++q) {
                const int32_t tq = tv + 32 * q;
                const int nv = min(32, seg.tok_end - tq);
                if (nv <= 0) break;
                const int64_t row =
                    resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size, b, tq);
                if (row < 0 && lane == 0) record_status(MLA_ERR_DEVICE_FAULT);
                if (!wait0(c.bar(B_VEMPTY0 + stage), phase ^ 1)) return;
                const uint32_t full = c.leader_bar(B_VFULL0 + stage);
                const uint32_t dst = c.sbase + kOffV + stage * kVStage;
                const int32_t z0 = 4 * static_cast<int32_t>(c.rank);  // column block of latent column 256r
                if (row >= 0 && nv == 32) {
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx_cluster(full, kVStage);
                        ptx::tma_load_3d_pair(dst, tm_v, 0, static_cast<int32_t>(row), z0, full);
                    }
                } else {
                    // Tail of the visible range: rows past it may hold anything (even NaN),
                    // and 0 * NaN would poison O, so they are zeroed before the MMA reads them.
                    int keep = 0;
                    if (row >= 0) {
                        if (lane == 0) {
                            ptx::mbar_arrive_expect_tx_local(c.bar(B_PATCH), kVStage);
                            ptx::tma_load_3d(dst, tm_v, 0, static_cast<int32_t>(row), z0, c.bar(B_PATCH));
                        }
                        if (!wait0(c.bar(B_PATCH), patch_phase)) return;
                        patch_phase ^= 1;
                        keep = nv;
                    }
                    uint4* p = reinterpret_cast<uint4*>(c.smem + kOffV + stage * kVStage);
                    for (int i = static_cast<int>(lane); i < kVStage / 16; i += 32) {
                        const int r = (i & 255) >> 3;  // token row within its 4 KB box
                        if (r >= keep) p[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive_cluster(full);
                }
                ring_next<kVStages>(stage, phase);
            }
        }
    }
    for (int i = 0; i < kVStages; ++i) {  // tail, as for the key ring
        if (!wait0(c.bar(B_VEMPTY0 + stage), phase ^ 1)) return;
        ring_next<kVStages>(stage, phase);
    }
}

// ------------------------------------------------------------ FP8 cache loads
// Coordinates of pool row `row` (= block * block_size + slot) in the FP8 maps.
struct F8At {
    int32_t slot, block;
};
__device__ __forceinline__ F8At f8_at(int64_t row, int32_t bs) {
    return {static_cast<int32_t>(row % bs), static_cast<int32_t>(row / bs)};
}

// Queries and key stages over the FP8 cache; one thread (lane 0 of warp 0).
// tm_k8: the codes {640 bytes, block_size rows, blocks} (row pitch 640, block
// pitch f8_block_bytes), box {64, 64, 1}, unswizzled; tm_ks: the scales
// {block_size, blocks} fp32, box {64, 1}; tm_kr: the f16 RoPE keys {64,
// block_size, blocks}, box {64, 64, 1}, 128B-swizzled. Key stage ks receives
// the codes of its column blocks (all but block 8, the RoPE key) in the upper
// halves of their boxes, the page's 64 scales at the start of its first box,
// and (last stage) the RoPE box in place, all on this CTA's KRAW barrier; the
// key expansion warp then fills the leader's KFULL.
__device__ void key_producer_f8(const Params& P, const CUtensorMap* tm_q, const CUtensorMap* tm_k8,
                                const CUtensorMap* tm_ks, const CUtensorMap* tm_kr, const Ctx& c) {
    uint32_t phase = 0;
    int seg_i = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    {
        SegmentIter peek = it;
        if (peek.next(seg)) prefetch_page<true>(P, c, seg, 0);
    }
    while (it.next(seg)) {
        const int32_t g = seg.group, b = g / P.q_len;
        if (seg_i > 0 && !ptx::mbar_wait(c.bar(B_QEMPTY), (seg_i - 1) & 1, c.abort, c.wait_ns)) return;
        {
            const uint32_t full = c.leader_bar(B_QFULL);
            ptx::mbar_arrive_expect_tx_cluster(full, kQBoxes * kBox);
            ptx::tma_load_3d_pair(c.sbase + kOffQ, tm_q, 0, g * kH + 64 * c.rank, 0, full);
        }
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const int32_t t0 = seg.tok_begin + j * kTile;
            int32_t th = t0 + 64 * static_cast<int32_t>(c.rank);
            if (th >= seg.tok_end) th = t0;  // no visible token in this half: any valid page (masked)
            int64_t row = resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size,
                                      b, th);
            if (row < 0) {
                record_status(MLA_ERR_DEVICE_FAULT);
                row = 0;
            }
            const F8At at = f8_at(row, P.block_size);
            if (j + 1 < n_tiles) {
                prefetch_page<true>(P, c, seg, j + 1);
            } else {
                SegmentIter peek = it;
                Segment nx;
                if (peek.next(nx)) prefetch_page<true>(P, c, nx, 0);
            }
            for (int ks = 0; ks < kKStages; ++ks) {
                if (!ptx::mbar_wait(c.bar(B_KEMPTY0 + ks), phase ^ 1, c.abort, c.wait_ns)) return;
                const uint32_t raw = c.bar(B_KRAW0 + ks);
                const int blk = kstage_first_block(ks);
                const bool last = ks == kKStages - 1;
                const int n8 = last ? kstage_blocks(ks) - 1 : kstage_blocks(ks);
                ptx::mbar_arrive_expect_tx_local(raw, n8 * kF8KSrc + 64 * 4 + (last ? kBox : 0));
                for (int i = 0; i < n8; ++i)
                    ptx::tma_load_3d(c.sbase + kOffK + (blk + i) * kBox + kF8KSrc, tm_k8, 64 * (blk + i), at.slot,
                                     at.block, raw);
                ptx::tma_load_2d(c.sbase + kOffK + blk * kBox, tm_ks, at.slot, at.block, raw);
                if (last) ptx::tma_load_3d(c.sbase + kOffK + (kQBoxes - 1) * kBox, tm_kr, 0, at.slot, at.block, raw);
            }
            phase ^= 1;
        }
        ++seg_i;
    }
    for (int ks = 0; ks < kKStages; ++ks)  // tail, as in key_producer
        if (!ptx::mbar_wait(c.bar(B_KEMPTY0 + ks), phase ^ 1, c.abort, c.wait_ns)) return;
    if (seg_i > 0) ptx::mbar_wait(c.bar(B_QEMPTY), (seg_i - 1) & 1, c.abort, c.wait_ns);
}

// Value stages over the FP8 cache; one thread (lane 0 of warp 2). tm_v8: the
// codes with box {64, 32, 1}; tm_vs: the scales with box {32, 1}. Stage q of a
// tile (tokens 32q..32q+31; box bx = latent columns 256r + 64bx) receives the
// codes of its four boxes in their upper halves and the 32 scales at its start,
// on this CTA's VRAW barrier; rows past the visible range are loaded too and
// zeroed by the value expansion warp, which then fills the leader's VFULL.
__device__ void value_producer_f8(const Params& P, const CUtensorMap* tm_v8, const CUtensorMap* tm_vs, const Ctx& c) {
    uint32_t stage = 0, phase = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        const int32_t b = seg.group / P.q_len;
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const int32_t tv = seg.tok_begin + j * kTile;
            for (int q = 0; q < kVPerTile; ++q) {
                const int32_t tq = tv + 32 * q;
                if (seg.tok_end - tq <= 0) break;
                const int64_t row =
                    resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size, b, tq);
                if (!ptx::mbar_wait(c.bar(B_VEMPTY0 + stage), phase ^ 1, c.abort, c.wait_ns)) return;
                const uint32_t raw = c.bar(B_VRAW0 + stage);
                const uint32_t dst = c.sbase + kOffV + stage * kVStage;
                if (row >= 0) {
                    const F8At at = f8_at(row, P.block_size);
                    ptx::mbar_arrive_expect_tx_local(raw, 4 * kF8VSrc + 32 * 4);
                    for (int bx = 0; bx < 4; ++bx)
                        ptx::tma_load_3d(dst + bx * (kBox / 2) + kF8VSrc, tm_v8,
                                         64 * (4 * static_cast<int32_t>(c.rank) + bx), at.slot, at.block, raw);
                    ptx::tma_load_2d(dst, tm_vs, at.slot, at.block, raw);
                } else {
                    record_status(MLA_ERR_DEVICE_FAULT);
                    ptx::mbar_arrive_local(raw);  // nothing loaded: the expansion writes zeros
                }
                ring_next<kVStages>(stage, phase);
            }
        }
    }
    for (int i = 0; i < kVStages; ++i) {  // tail, as for the key ring
        if (!ptx::mbar_wait(c.bar(B_VEMPTY0 + stage), phase ^ 1, c.abort, c.wait_ns)) return;
        ring_next<kVStages>(stage, phase);
    }
}

// A wait by every lane of a warp that succeeds for all of them or for none (a
// lane that gave up makes its warp give up): warp-collective code after it
// (tensor-memory loads and stores, __syncwarp) stays converged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, limit_ns));
}

// One box expanded in place by a warp: rows r0 + 8k (k < K; r0 = lane / 4) of
// 64 codes at `src` (64-byte rows; this lane's 16-byte chunk ch = lane % 4)
// become f16 rows of 128 bytes at `box` in the TMA's SWIZZLE_128B layout
// (16-byte chunk i of row r at position i ^ (r % 8); the box is 1 KB aligned),
// the two chunks of this lane being 2ch and 2ch + 1. Rows >= keep become
// zeros. s2[k]: the f16x2 scale of row r0 + 8k. Every lane reads its codes
// before any lane writes, since rows 32.. of the box overlay the codes.
template <int K>
__device__ __forceinline__ void expand_box(uint8_t* box, const uint8_t* src, const uint32_t (&s2)[K], int r0,
                                           int ch, int keep) {
    uint4 v[K];
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = *reinterpret_cast<const uint4*>(src + (r0 + 8 * k) * 64 + 16 * ch);
    __syncwarp();
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int r = r0 + 8 * k;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (r < keep) {
            const uint2 a = fp8::dequant4(v[k].x, s2[k]), b = fp8::dequant4(v[k].y, s2[k]);
            const uint2 d = fp8::dequant4(v[k].z, s2[k]), e = fp8::dequant4(v[k].w, s2[k]);
            lo = make_uint4(a.x, a.y, b.x, b.y);
            hi = make_uint4(d.x, d.y, e.x, e.y);
        }
        uint8_t* rowp = box + r * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * ch) ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(rowp + (((2 * ch + 1) ^ (r & 7)) << 4)) = hi;
    }
}

// Key expansion (warp 10): per tile and key stage, after KRAW, the stage's
// code boxes become f16 key boxes (scales read first: they sit in the first
// box), then the stage is signalled to the leader's KFULL (count 2: both CTAs).
__device__ void key_expander(const Params& P, const Ctx& c) {
    const uint32_t lane = ptx::lane_id();
    const int r0 = static_cast<int>(lane >> 2), ch = static_cast<int>(lane & 3);
    uint32_t phase = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            for (int ks = 0; ks < kKStages; ++ks) {
                if (!warp_wait(c.bar(B_KRAW0 + ks), phase, c.abort, c.wait_ns)) return;
                const int blk = kstage_first_block(ks);
                const int n8 = ks == kKStages - 1 ? kstage_blocks(ks) - 1 : kstage_blocks(ks);
                const float* sc = reinterpret_cast<const float*>(c.smem + kOffK + blk * kBox);
                uint32_t s2[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) s2[k] = fp8::scale_f16x2(sc[r0 + 8 * k]);
#pragma unroll 1
                for (int i = 0; i < n8; ++i) {
                    uint8_t* box = c.smem + kOffK + (blk + i) * kBox;
                    expand_box<8>(box, box + kF8KSrc, s2, r0, ch, 64);
                }
                ptx::fence_proxy_async_smem();  // the generic-proxy writes, before the MMAs read them
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(c.leader_bar(B_KFULL0 + ks));
            }
            phase ^= 1;
        }
    }
}

// Value expansion (warp 11): per visible value stage, after VRAW, its four code
// boxes become f16 value boxes (rows past the visible range, or all rows if the
// page is missing, as zeros), then VFULL of the leader (count 2).
__device__ void value_expander(const Params& P, const Ctx& c) {
    const uint32_t lane = ptx::lane_id();
    const int r0 = static_cast<int>(lane >> 2), ch = static_cast<int>(lane & 3);
    uint32_t stage = 0, phase = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        const int32_t b = seg.group / P.q_len;
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const int32_t tv = seg.tok_begin + j * kTile;
            for (int q = 0; q < kVPerTile; ++q) {
                const int32_t tq = tv + 32 * q;
                const int nv = min(32, seg.tok_end - tq);
                if (nv <= 0) break;
                const int64_t row =
                    resolve_row(P.block_table, P.batch, P.max_blocks_per_seq, P.num_blocks, P.block_size, b, tq);
                if (!warp_wait(c.bar(B_VRAW0 + stage), phase, c.abort, c.wait_ns)) return;
                const int keep = row >= 0 ? nv : 0;
                uint8_t* st = c.smem + kOffV + stage * kVStage;
                const float* sc = reinterpret_cast<const float*>(st);
                uint32_t s2[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) s2[k] = fp8::scale_f16x2(sc[r0 + 8 * k]);
#pragma unroll 1
                for (int bx = 0; bx < 4; ++bx) {
                    uint8_t* box = st + bx * (kBox / 2);
                    expand_box<4>(box, box + kF8VSrc, s2, r0, ch, keep);
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(c.leader_bar(B_VFULL0 + stage));
                ring_next<kVStages>(stage, phase);
            }
        }
    }
}

// ------------------------------------------------------------------- MMA
// Four issuing threads in the leader CTA: two for the score MMAs, two for the
// value MMAs. A single thread issues at most about one tcgen05.mma every ~47
// cycles, while an M 128 x N 128 x K 16 pair instruction takes the tensor
// cores 32 cycles; streams with their own accumulators keep up together.
struct Descs {
    uint64_t dq, dk, dp, dv;
    __device__ explicit Descs(const Ctx& c)
        // base descriptors; operand offsets are added in 16-byte units to the start-address field
        : dq(ptx::smem_desc_sw128(c.sbase + kOffQ, 16, 1024)),
          dk(ptx::smem_desc_sw128(c.sbase + kOffK, 16, 1024)),
          dp(ptx::smem_desc_sw128(c.sbase + kOffP, 16, 1024)),
          dv(ptx::smem_desc_sw128(c.sbase + kOffV, kBox / 2, 1024)) {}
};

// Score MMAs, half h (lane 0 of warp 1: h = 0; lane 0 of warp 3: h = 1):
// S_h = Q[:, blocks] K[:, blocks]^T over column blocks 0-4 (key stages 0-1) or
// 5-8 (stages 2-3) into half-accumulator h of S buffer (tile & 1), up to two
// tiles ahead of the softmax (the S buffers). Each key stage is consumed by
// one thread, once per tile (phase = tile parity); both threads commit QEMPTY
// (count 2) once per segment and SFULL (count 2) once per tile. kF16: f16
// operands (FP8 cache) instead of bf16.
template <bool kF16>
__device__ void mma_s_issuer(const Params& P, const Ctx& c, uint32_t half) {
    constexpr uint32_t kIdS = kF16 ? ptx::idesc_f16(128, 128, false, false) : ptx::idesc_bf16(128, 128, false, false);
    const Descs D(c);
    uint32_t tile_cnt = 0;
    int seg_i = 0;
    const int ks0 = 2 * static_cast<int>(half);
    const int k_first = kstage_first_block(ks0);
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        if (!ptx::mbar_wait(c.bar(B_QFULL), seg_i & 1, c.abort, c.wait_ns)) return;
        ptx::tc_fence_after();
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j, ++tile_cnt) {
            const uint32_t sb = tile_cnt & 1;
            const uint32_t d_s = c.tmem + kTmS + 128 * sb + 64 * half;
            if (!ptx::mbar_wait(c.bar(B_SEMPTY0 + sb), ((tile_cnt >> 1) & 1) ^ 1, c.abort, c.wait_ns)) return;
#pragma unroll 1
            for (int ks = ks0; ks < ks0 + 2; ++ks) {
                if (!ptx::mbar_wait(c.bar(B_KFULL0 + ks), tile_cnt & 1, c.abort, c.wait_ns)) return;
                ptx::tc_fence_after();
                for (int k = kstage_first_block(ks); k < kstage_first_block(ks) + kstage_blocks(ks); ++k) {
                    const uint64_t a0 = D.dq + static_cast<uint64_t>((k * kBox) >> 4);
                    const uint64_t b0 = D.dk + static_cast<uint64_t>((k * kBox) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::mma_bf16_pair(d_s, a0 + 2 * kk, b0 + 2 * kk, kIdS, (k != k_first) || (kk != 0));
                }
                ptx::mma_commit_pair(c.bar(B_KEMPTY0 + ks), 0x3);
            }
            ptx::mma_commit_pair(c.bar(B_SFULL0 + sb), 0x3);
        }
        ptx::mma_commit_pair(c.bar(B_QEMPTY), 0x3);
        ++seg_i;
    }
}

// Value MMAs, half h (lane 0 of warp 8 + h): O[:, 256h .. 256h + 255] += P V
// over the tile's visible 32-token value stages (stage q: tokens 32q..32q+31,
// stages without a visible token skipped here and by the producer alike).
// Both threads read every value stage and commit its VEMPTY (count 2), and
// PVDONE (count 2) once per tile. The first value MMA of a segment overwrites
// O, after the softmax has read out the previous segment (OEMPTY).
template <bool kF16>
__device__ void mma_pv_issuer(const Params& P, const Ctx& c, uint32_t half) {
    constexpr uint32_t kIdPV = kF16 ? ptx::idesc_f16(128, 256, false, true) : ptx::idesc_bf16(128, 256, false, true);
    const Descs D(c);
    uint32_t vst = 0, vph = 0, pv_cnt = 0;
    int seg_i = 0;
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const bool first = (j == 0);
            if (!ptx::mbar_wait(c.bar(B_PFULL0 + (pv_cnt & 1)), (pv_cnt >> 1) & 1, c.abort, c.wait_ns)) return;
            if (first && !ptx::mbar_wait(c.bar(B_OEMPTY), (seg_i & 1) ^ 1, c.abort, c.wait_ns)) return;
            const int32_t tv = seg.tok_begin + j * kTile;
            for (int q = 0; q < kVPerTile; ++q) {
                if (seg.tok_end - (tv + 32 * q) <= 0) break;
                if (!ptx::mbar_wait(c.bar(B_VFULL0 + vst), vph, c.abort, c.wait_ns)) return;
                ptx::tc_fence_after();
                const uint64_t a0 = D.dp + static_cast<uint64_t>(((q >> 1) * kBox + 64 * (q & 1)) >> 4);
                const uint64_t b0 = D.dv + static_cast<uint64_t>((vst * kVStage + half * kBox) >> 4);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    ptx::mma_bf16_pair(c.tmem + kTmO + 128 * half, a0 + 2 * kk,
                                       b0 + static_cast<uint64_t>((2048 * kk) >> 4), kIdPV,
                                       !(first && q == 0 && kk == 0));
                ptx::mma_commit_pair(c.bar(B_VEMPTY0 + vst), 0x3);
                ring_next<kVStages>(vst, vph);
            }
            ptx::mma_commit_pair(c.bar(B_PVDONE0 + (pv_cnt & 1)), 0x3);
            ++pv_cnt;
        }
        ++seg_i;
    }
}

// --------------------------------------------------------------- softmax
// The softmax warps execute warp-collective tensor-memory instructions
// (tcgen05.ld / st .sync.aligned), so every branch they take must be
// warp-uniform: waits go through warp_wait, and the O rescale runs for the
// whole warp when any of its rows needs it.

struct Exchanger {  // swaps one float between thread t and thread t ^ 64 of the softmax warps
    float* red;
    uint32_t bar;
    uint32_t n = 0;
    __device__ bool swap(float v, float& partner, int t, volatile int* abort, uint64_t limit_ns) {
        float* buf = red + (n & 1) * 128;
        buf[t] = v;
        __syncwarp();
        if (ptx::lane_id() == 0) ptx::mbar_arrive_local(bar);
        if (!warp_wait(bar, n & 1, abort, limit_ns)) return false;
        partner = buf[t ^ 64];
        ++n;
        return true;
    }
};

template <bool kF16>
__device__ void softmax(const Params& P, const Ctx& c) {
    const int t = static_cast<int>(threadIdx.x) - 128;  // TMEM lane
    const uint32_t lane = ptx::lane_id();
    const int half = t >> 6, hrow = t & 63;
    const int head = 64 * static_cast<int>(c.rank) + hrow;
    const uint32_t tl = c.tmem + (static_cast<uint32_t>(t & ~31) << 16);  // this warp's lane quadrant
    const uint32_t sempty0 = c.leader_bar(B_SEMPTY0), sempty1 = c.leader_bar(B_SEMPTY1);
    const float scale_log2 = P.scale_log2;
    const uint32_t pfull0 = c.leader_bar(B_PFULL0), pfull1 = c.leader_bar(B_PFULL1);
    const uint32_t oempty = c.leader_bar(B_OEMPTY);
    Exchanger xc{reinterpret_cast<float*>(c.smem + kOffRed), c.bar(B_XCHG)};
    uint32_t tile_cnt = 0;
    // Value MMAs of the pair's tile k signal PVDONE[k & 1] (phase k >> 1). pv_done is the
    // highest k known complete (a completion implies every earlier one). Each wait is at
    // most one phase behind its barrier: tile k + 1's value MMAs need the P this thread
    // writes after the wait.
    int32_t pv_done = -1;
    auto wait_pv = [&](int32_t k) -> bool {
        if (k <= pv_done) return true;
        if (!warp_wait(c.bar(B_PVDONE0 + (k & 1)), (static_cast<uint32_t>(k) >> 1) & 1, c.abort, c.wait_ns)) return false;
        pv_done = k;
        return true;
    };
    SegmentIter it(P.hdr, P.worker_group, P.tile_prefix, P.part_offsets, P.context_lens, P.q_len, kTile, c.pair);
    Segment seg;
    while (it.next(seg)) {
        float m_run = -INFINITY, l_run = 0.f;
        const int n_tiles = tiles_of(seg);
        for (int j = 0; j < n_tiles; ++j) {
            const int32_t tc = static_cast<int32_t>(tile_cnt);
            const uint32_t sb = tile_cnt & 1;
            if (!warp_wait(c.bar(B_SFULL0 + sb), (tile_cnt >> 1) & 1, c.abort, c.wait_ns)) return;
            ptx::tc_fence_after();
            float s[64];
            {
                float (&s0)[32] = *reinterpret_cast<float(*)[32]>(&s[0]);
                float (&s1)[32] = *reinterpret_cast<float(*)[32]>(&s[32]);
                ptx::tmem_ld32(tl + kTmS + 128 * sb, s0);
                ptx::tmem_ld32(tl + kTmS + 128 * sb + 32, s1);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {  // + the hi half-accumulator
                    float u[32];
                    ptx::tmem_ld32(tl + kTmS + 128 * sb + 64 + 32 * h2, u);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[32 * h2 + i] += u[i];
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(sb ? sempty1 : sempty0);
            ++tile_cnt;

            const int32_t tok0 = seg.tok_begin + j * kTile + 64 * half;
            const int nvalid = max(0, min(64, seg.tok_end - tok0));
            if (nvalid < 64) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (i >= nvalid) s[i] = -INFINITY;
            }
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], s[i]);
            // the scale is positive, so the max of the raw scores gives the max of the scaled ones
            const float mloc = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
            float mpart;
            if (!xc.swap(mloc, mpart, t, c.abort, c.wait_ns)) return;
            const float m_tile = fmaxf(mloc, mpart);
            const float m_new = fmaxf(m_run, m_tile);
            const bool rescale = m_new > m_run + 8.f;  // keep a stale max unless it grows by > 2^8
            const float m_use = rescale ? m_new : m_run;
            const float alpha = rescale ? ptx::ex2(m_run - m_new) : 1.f;
            const float neg_m = -m_use;
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                s[i] = ptx::ex2(fmaf(s[i], scale_log2, neg_m));  // 2^-inf = 0 for masked tokens
                ps[i & 3] += s[i];
            }
            l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
            // O is rescaled once the previous tile's value MMAs are done, by the whole warp
            // (alpha = 1 in the rows that keep their max)
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                if (!wait_pv(tc - 1)) return;
                ptx::tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    float o[32];
                    ptx::tmem_ld32(tl + kTmO + 32 * cc, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    ptx::tmem_st32(tl + kTmO + 32 * cc, o);
                }
                ptx::tmem_wait_st();
            }
            // the P buffer was last read by the value MMAs of tile tc - 1
            if (tc >= 1 && !wait_pv(tc - 1)) return;
            ptx::tc_fence_after();
            uint8_t* const prow = c.smem + kOffP + half * kBox + hrow * 128;
            // P row (bf16, or f16 with the FP8 cache) into the K-major 128B-swizzled A
            // operand of the PV MMA
            auto pk = [](float lo, float hi) { return kF16 ? ptx::f16x2(lo, hi) : ptx::bf16x2(lo, hi); };
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                uint4 u;
                u.x = pk(s[8 * c8 + 0], s[8 * c8 + 1]);
                u.y = pk(s[8 * c8 + 2], s[8 * c8 + 3]);
                u.z = pk(s[8 * c8 + 4], s[8 * c8 + 5]);
                u.w = pk(s[8 * c8 + 6], s[8 * c8 + 7]);
                *reinterpret_cast<uint4*>(prow + ((c8 ^ (hrow & 7)) << 4)) = u;
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(sb ? pfull1 : pfull0);
            m_run = m_use;
        }
        // segment epilogue: normalise O and write the partial
        if (!wait_pv(static_cast<int32_t>(tile_cnt) - 1)) return;
        ptx::tc_fence_after();
        float lpart;
        if (!xc.swap(l_run, lpart, t, c.abort, c.wait_ns)) return;
        const float l_tot = l_run + lpart;
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        // O rows go out, rounded to bf16, through the (now idle) P buffers: each thread
        // writes a 64-column slice of its row (128 bytes, 16-byte chunks XOR-swizzled
        // by row) to shared memory, then the warp stores its 32 rows with 8 lanes per
        // 128-byte row segment, so every global store instruction covers whole lines.
        uint16_t* const o_base = P.o_part + static_cast<int64_t>(seg.slot) * kH * kDc;
        uint8_t* const stage_buf = c.smem + kOffP;
        const int wrow0 = t & ~31;  // first row (thread) of this warp
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            float o[64];
            {
                float (&o0)[32] = *reinterpret_cast<float(*)[32]>(&o[0]);
                float (&o1)[32] = *reinterpret_cast<float(*)[32]>(&o[32]);
                ptx::tmem_ld32(tl + kTmO + 64 * cc, o0);
                ptx::tmem_ld32(tl + kTmO + 64 * cc + 32, o1);
                ptx::tmem_wait_ld();
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint4 u;
                u.x = ptx::bf16x2(o[8 * k + 0] * inv, o[8 * k + 1] * inv);
                u.y = ptx::bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv);
                u.z = ptx::bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv);
                u.w = ptx::bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv);
                *reinterpret_cast<uint4*>(stage_buf + t * 128 + ((k ^ (t & 7)) << 4)) = u;
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int r = wrow0 + 4 * k + static_cast<int>(lane >> 3), ch = static_cast<int>(lane & 7);
                const uint4 v = *reinterpret_cast<const uint4*>(stage_buf + r * 128 + ((ch ^ (r & 7)) << 4));
                const int r_head = 64 * static_cast<int>(c.rank) + (r & 63);
                *reinterpret_cast<uint4*>(o_base + static_cast<int64_t>(r_head) * kDc + 256 * (r >> 6) + 64 * cc +
                                          8 * ch) = v;
            }
            __syncwarp();
        }
        if (half == 0)
            P.lse_part[static_cast<int64_t>(seg.slot) * kH + head] =
                l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(oempty);
    }
}

// ------------------------------------------------------------------ kernel
// grid: 2 * workers CTAs (clusters of 2); block kThreads; dynamic smem kSmemBytes.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    pair_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k3,
                       const __grid_constant__ CUtensorMap tm_k2, const __grid_constant__ CUtensorMap tm_v,
                       const Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5;
    Ctx c;
    c.smem = smem;
    c.sbase = ptx::smem_u32(smem);
    c.rank = ptx::cluster_ctarank();
    c.pair = ptx::cluster_id_x();
    c.abort = reinterpret_cast<volatile int*>(smem + kOffMisc);
    c.wait_ns = P.wait_ns;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc + 16);

    if (threadIdx.x == 0) {
        *c.abort = 0;
        ptx::mbar_init(c.bar(B_QFULL), 2);
        ptx::mbar_init(c.bar(B_QEMPTY), 2);
        ptx::mbar_init(c.bar(B_SFULL0), 2);
        ptx::mbar_init(c.bar(B_SFULL1), 2);
        ptx::mbar_init(c.bar(B_SEMPTY0), 8);
        ptx::mbar_init(c.bar(B_SEMPTY1), 8);
        ptx::mbar_init(c.bar(B_PFULL0), 8);
        ptx::mbar_init(c.bar(B_PFULL1), 8);
        ptx::mbar_init(c.bar(B_PVDONE0), 2);
        ptx::mbar_init(c.bar(B_PVDONE1), 2);
        ptx::mbar_init(c.bar(B_OEMPTY), 8);
        ptx::mbar_init(c.bar(B_PATCH), 1);
        ptx::mbar_init(c.bar(B_XCHG), 4);
        for (int s = 0; s < kKStages; ++s) {
            ptx::mbar_init(c.bar(B_KFULL0 + s), 2);
            ptx::mbar_init(c.bar(B_KEMPTY0 + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            ptx::mbar_init(c.bar(B_VFULL0 + s), 2);
            ptx::mbar_init(c.bar(B_VEMPTY0 + s), 2);
        }
        ptx::fence_mbar_init();
    }
    if (warp == 0 && ptx::lane_id() == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k3);
        ptx::prefetch_tmap(&tm_k2);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // the peer's barriers exist before anyone arrives on them
    ptx::tc_fence_after();
    c.tmem = *tmem_slot;
    pdl_wait();  // the schedule and the absorbed queries come from the preceding kernels
    pdl_trigger();

    if (warp == 0) {
        if (ptx::lane_id() == 0 && !P.starve) key_producer(P, &tm_q, &tm_k3, &tm_k2, c);
    } else if (warp == 2) {
        if (!P.starve) value_producer(P, &tm_v, c);
    } else if (warp == 1 || warp == 3) {
        if (c.rank == 0 && ptx::lane_id() == 0) mma_s_issuer<false>(P, c, static_cast<uint32_t>(warp >> 1));
    } else if (warp >= 8) {
        if (c.rank == 0 && ptx::lane_id() == 0) mma_pv_issuer<false>(P, c, static_cast<uint32_t>(warp - 8));
    } else if (warp >= 4) {
        softmax<false>(P, c);
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // no MMA or remote arrive targets this CTA any more
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(c.tmem, kTmemCols);
    }
}

// The same kernel over the FP8 cache: f16 queries and softmax weights, the
// cache boxes expanded in place by warps 10 and 11 (see the header). grid: 2 *
// workers CTAs (clusters of 2); block kF8Threads; dynamic smem kSmemBytes.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kF8Threads, 1)
    pair_decode_f8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                          const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_kr,
                          const __grid_constant__ CUtensorMap tm_v8, const __grid_constant__ CUtensorMap tm_vs,
                          const Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5;
    Ctx c;
    c.smem = smem;
    c.sbase = ptx::smem_u32(smem);
    c.rank = ptx::cluster_ctarank();
    c.pair = ptx::cluster_id_x();
    c.abort = reinterpret_cast<volatile int*>(smem + kOffMisc);
    c.wait_ns = P.wait_ns;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc + 16);

    if (threadIdx.x == 0) {
        *c.abort = 0;
        ptx::mbar_init(c.bar(B_QFULL), 2);
        ptx::mbar_init(c.bar(B_QEMPTY), 2);
        ptx::mbar_init(c.bar(B_SFULL0), 2);
        ptx::mbar_init(c.bar(B_SFULL1), 2);
        ptx::mbar_init(c.bar(B_SEMPTY0), 8);
        ptx::mbar_init(c.bar(B_SEMPTY1), 8);
        ptx::mbar_init(c.bar(B_PFULL0), 8);
        ptx::mbar_init(c.bar(B_PFULL1), 8);
        ptx::mbar_init(c.bar(B_PVDONE0), 2);
        ptx::mbar_init(c.bar(B_PVDONE1), 2);
        ptx::mbar_init(c.bar(B_OEMPTY), 8);
        ptx::mbar_init(c.bar(B_PATCH), 1);
        ptx::mbar_init(c.bar(B_XCHG), 4);
        for (int s = 0; s < kKStages; ++s) {
            ptx::mbar_init(c.bar(B_KFULL0 + s), 2);   // the key expansion warps of both CTAs
            ptx::mbar_init(c.bar(B_KEMPTY0 + s), 1);
            ptx::mbar_init(c.bar(B_KRAW0 + s), 1);    // this CTA's producer (+ its copies' bytes)
        }
        for (int s = 0; s < kVStages; ++s) {
            ptx::mbar_init(c.bar(B_VFULL0 + s), 2);   // the value expansion warps of both CTAs
            ptx::mbar_init(c.bar(B_VEMPTY0 + s), 2);
            ptx::mbar_init(c.bar(B_VRAW0 + s), 1);
        }
        ptx::fence_mbar_init();
    }
    if (warp == 0 && ptx::lane_id() == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k8);
        ptx::prefetch_tmap(&tm_ks);
        ptx::prefetch_tmap(&tm_kr);
        ptx::prefetch_tmap(&tm_v8);
        ptx::prefetch_tmap(&tm_vs);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // the peer's barriers exist before anyone arrives on them
    ptx::tc_fence_after();
    c.tmem = *tmem_slot;
    pdl_wait();  // the schedule and the absorbed queries come from the preceding kernels
    pdl_trigger();

    if (warp == 0) {
        if (ptx::lane_id() == 0 && !P.starve) key_producer_f8(P, &tm_q, &tm_k8, &tm_ks, &tm_kr, c);
    } else if (warp == 2) {
        if (ptx::lane_id() == 0 && !P.starve) value_producer_f8(P, &tm_v8, &tm_vs, c);
    } else if (warp == 1 || warp == 3) {
        if (c.rank == 0 && ptx::lane_id() == 0) mma_s_issuer<true>(P, c, static_cast<uint32_t>(warp >> 1));
    } else if (warp == 8 || warp == 9) {
        if (c.rank == 0 && ptx::lane_id() == 0) mma_pv_issuer<true>(P, c, static_cast<uint32_t>(warp - 8));
    } else if (warp == 10) {
        key_expander(P, c);
    } else if (warp == 11) {
        value_expander(P, c);
    } else {
        softmax<true>(P, c);
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // no MMA or remote arrive targets this CTA any more
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(c.tmem, kTmemCols);
    }
}

}  // namespace pair
}  // namespace mla
