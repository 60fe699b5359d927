// C ABI of the MLA decode library: argument validation, workspace layout and
// kernel launches. Every entry point returns an mla_status_t and never
// allocates, frees or synchronises (except mla_get_device_error, whose job
// is to synchronise and read the device status word).
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <utility>

#include "mla_b200.h"
#include "common.cuh"
#include "plan.cuh"
#include "absorb.cuh"
#include "combine.cuh"
#include "decode_generic.cuh"
#include "append.cuh"
#include "decode_pair.cuh"
#include "gemm_tc05.cuh"
#include "qproj.cuh"

#include <cudaTypedefs.h>

namespace mla {
namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Dims the CUDA-core kernels implement.
int check_dims(const mla_dims_t* d) {
    if (!d) return MLA_ERR_INVALID_ARG;
    if (d->num_heads < 1 || d->kv_lora_rank < 8 || d->rope_dim < 2 || d->qk_nope_dim < 1 ||
        d->v_head_dim < 1 || d->block_size < 1 || !(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale))
        return MLA_ERR_INVALID_ARG;
    if (d->num_heads > 1024 || d->kv_lora_rank > 16 * kGenMaxCols || d->rope_dim > 128 ||
        d->qk_nope_dim > 512 || d->v_head_dim > 512)
        return MLA_ERR_UNSUPPORTED_DIMS;
    if ((d->kv_lora_rank + d->rope_dim) % 8 != 0 || d->rope_dim % 2 != 0) return MLA_ERR_UNSUPPORTED_DIMS;
    return MLA_OK;
}

int device_ok() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MLA_ERR_NO_DEVICE; }
    static int cached[64] = {0};  // 0 unknown, 1 ok, 2 not sm_100
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] == 1 ? MLA_OK : MLA_ERR_NO_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_NO_DEVICE;
    }
    const int ok = major == 10 ? 1 : 2;
    if (dev >= 0 && dev < 64) cached[dev] = ok;
    return ok == 1 ? MLA_OK : MLA_ERR_NO_DEVICE;
}

// Launches `kernel` on `st` with programmatic stream serialization (the
// kernels call pdl_wait() before touching data of earlier work, see common.cuh).
template <typename... KArgs, typename... Args>
int launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, dim3 cluster,
                   Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster.x * cluster.y * cluster.z > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster.x;
        attr[1].val.clusterDim.y = cluster.y;
        attr[1].val.clusterDim.z = cluster.z;
        cfg.numAttrs = 2;
    }
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
    return launch_cluster(kernel, grid, block, smem, st, dim3(1, 1, 1), std::forward<Args>(args)...);
}

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// ---- decode workspace ------------------------------------------------
struct DecodeLayout {
    size_t hdr, tile_prefix, part_offsets, worker_group, q, o_part, lse_part, total;
    int32_t workers, max_parts, kernel, tile;
};

constexpr int kKernelPair = 1, kKernelGeneric = 2;

// The tensor-core pair kernel is specialised to DeepSeek-V3 dims and needs
// every 64-token half tile inside one page.
bool pair_kernel_fits(const mla_dims_t* d) {
    return d->num_heads == pair::kH && d->kv_lora_rank == pair::kDc && d->rope_dim == pair::kDr &&
           d->block_size % 64 == 0;
}

int pick_kernel(const mla_dims_t* d, const mla_decode_opts_t* o) {
    const int k = o ? o->kernel : 0;
    if (k == 0) return pair_kernel_fits(d) ? kKernelPair : kKernelGeneric;
    if (k == kKernelPair) return pair_kernel_fits(d) ? kKernelPair : -1;
    if (k == kKernelGeneric) return kKernelGeneric;
    return -1;
}

// G query groups of at most max_len visible tokens. The tensor-core kernel runs
// one cluster of two CTAs per SM pair, but a small problem is split no finer
// than about two 128-token tiles per worker: a worker's start-up (query load,
// pipeline fill) and its partial's write and merge cost about a tile, and two
// tiles let the loads of the second overlap the first (batch 1 x 4096 tokens:
// 43 us with 16 workers against 47 with 74).
int default_workers(const mla_dims_t* d, int kernel, int64_t G, int32_t max_len) {
    if (kernel == kKernelPair) {
        const int64_t tiles = G * ((static_cast<int64_t>(max_len) + pair::kTile - 1) / pair::kTile);
        return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms() / 2, (tiles + 1) / 2)));
    }
    const int hb = (d->num_heads + kGenHeads - 1) / kGenHeads;
    const int target = 4 * num_sms();
    return target / hb > 0 ? target / hb : 1;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 3-D bf16 tensor map over rows of `cols` values seen as {64 columns, rows,
// cols / 64 column blocks} (row stride cols * 2 bytes, block stride 128 bytes),
// box = {64, box_rows, box_blocks}, 128-byte swizzle. A box lands in shared
// memory as box_blocks consecutive [box_rows x 64] swizzled tiles, the same
// bytes as box_blocks separate 2-D boxes of 64 columns.
int encode_row_blocks(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                      uint32_t box_blocks) {
    auto fn = tensor_map_encoder();
    if (!fn) return MLA_ERR_CUDA;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 2-D bf16 tensor map over a row-major matrix [rows, cols] (row stride `cols`
// * 2 bytes), box = {64 columns, box_rows rows}, 128-byte swizzle; rows past
// the end are zero-filled.
int encode_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    auto fn = tensor_map_encoder();
    if (!fn) return MLA_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 3-D bf16 tensor map over the split-KV partials [slots][H][d_c]: box {64
// columns, 1 head, 64 slots}, 128-byte swizzle; slots past the end read 0.
int encode_parts(CUtensorMap* m, const void* base, uint64_t dc, uint64_t H, uint64_t slots) {
    auto fn = tensor_map_encoder();
    if (!fn) return MLA_ERR_CUDA;
    cuuint64_t dims[3] = {dc, H, slots};
    cuuint64_t strides[2] = {dc * 2, H * dc * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// A tiled tensor map of any rank (<= 3) and element type: dims / byte strides /
// box as cuTensorMapEncodeTiled takes them, unit element strides, L2
// promotion 256 B, no fill.
int encode_tiled(CUtensorMap* m, CUtensorMapDataType type, uint32_t rank, const void* base, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
    auto fn = tensor_map_encoder();
    if (!fn) return MLA_ERR_CUDA;
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, type, rank, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// The five maps of the FP8 cache the attention reads (fp8.cuh layout): codes
// {row bytes, block_size, blocks} with boxes {64, 64, 1} (keys) and {64, 32, 1}
// (values), unswizzled; the fp32 scales {block_size, blocks} with boxes
// {64, 1} and {32, 1}; the f16 RoPE keys {64, block_size, blocks} with box
// {64, 64, 1}, 128B-swizzled.
struct F8Maps {
    CUtensorMap k8, ks, kr, v8, vs;
};
int encode_f8_maps(F8Maps* M, const void* pool, const mla_dims_t* d, int64_t num_blocks) {
    const uint64_t rb = static_cast<uint64_t>(fp8::row_bytes(d->kv_lora_rank, d->rope_dim));
    const uint64_t bb = static_cast<uint64_t>(fp8::block_bytes(d->kv_lora_rank, d->rope_dim, d->block_size));
    const uint64_t bs = static_cast<uint64_t>(d->block_size), nb = static_cast<uint64_t>(num_blocks);
    const char* base = static_cast<const char*>(pool);
    {
        cuuint64_t dims[3] = {rb, bs, nb};
        cuuint64_t strides[2] = {rb, bb};
        cuuint32_t kbox[3] = {64, 64, 1}, vbox[3] = {64, 32, 1};
        if (int rc = encode_tiled(&M->k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, kbox,
                                  CU_TENSOR_MAP_SWIZZLE_NONE)) return rc;
        if (int rc = encode_tiled(&M->v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, vbox,
                                  CU_TENSOR_MAP_SWIZZLE_NONE)) return rc;
    }
    {
        cuuint64_t dims[2] = {bs, nb};
        cuuint64_t strides[1] = {bb};
        cuuint32_t kbox[2] = {64, 1}, vbox[2] = {32, 1};
        const char* sc = base + bs * rb;
        if (int rc = encode_tiled(&M->ks, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, sc, dims, strides, kbox,
                                  CU_TENSOR_MAP_SWIZZLE_NONE)) return rc;
        if (int rc = encode_tiled(&M->vs, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, sc, dims, strides, vbox,
                                  CU_TENSOR_MAP_SWIZZLE_NONE)) return rc;
    }
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(d->rope_dim), bs, nb};
        cuuint64_t strides[2] = {rb, bb};
        cuuint32_t box[3] = {64, 64, 1};
        if (int rc = encode_tiled(&M->kr, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base + d->kv_lora_rank, dims, strides,
                                  box, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    }
    return MLA_OK;
}

// The FP8 cache layout needs 16-byte rows, blocks and offsets (d_c a multiple
// of 16, d_r of 8, block_size of 4).
bool fp8_dims_ok(const mla_dims_t* d) {
    return d->kv_lora_rank % 16 == 0 && d->rope_dim % 8 == 0 && d->block_size % 4 == 0;
}

// The tcgen05 absorb / merge / UV kernels: d_n a multiple of 64 up to 256, d_c
// a multiple of 256 up to 512, d_r a multiple of 8 up to 64, d_v a multiple of 16 up
// to 256, and 16-byte aligned operands.
bool tc05_dims_ok(const mla_dims_t* d) {
    return d->qk_nope_dim % 64 == 0 && d->qk_nope_dim <= 256 && d->kv_lora_rank % 256 == 0 &&
           d->kv_lora_rank <= 512 && d->rope_dim % 8 == 0 && d->rope_dim <= 64 && d->v_head_dim % 16 == 0 &&
           d->v_head_dim <= 256;
}

int decode_layout(const mla_dims_t* d, int32_t batch, int32_t q_len, int32_t max_len,
                  const mla_decode_opts_t* o, DecodeLayout* L) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (batch < 1 || q_len < 1 || max_len < q_len) return MLA_ERR_INVALID_ARG;
    const int kernel = pick_kernel(d, o);
    if (kernel < 0) return MLA_ERR_UNSUPPORTED_DIMS;
    if (o && o->cache_fp8 && kernel != kKernelPair) return MLA_ERR_UNSUPPORTED_DIMS;  // only it reads FP8
    L->kernel = kernel;
    L->tile = kernel == kKernelPair ? pair::kTile : kGenTokens;
    const int64_t G = static_cast<int64_t>(batch) * q_len;
    const int64_t tiles_per_group = (max_len + L->tile - 1) / L->tile;
    if (G * tiles_per_group >= (int64_t(1) << 31) || G * d->num_heads >= (int64_t(1) << 31))
        return MLA_ERR_UNSUPPORTED_DIMS;
    int64_t workers = (o && o->num_workers > 0) ? o->num_workers : default_workers(d, kernel, G, max_len);
    if (workers > (int64_t(1) << 20)) workers = int64_t(1) << 20;
    L->workers = static_cast<int32_t>(workers);
    L->max_parts = static_cast<int32_t>(G + workers);
    const size_t D = static_cast<size_t>(d->kv_lora_rank) + d->rope_dim;
    size_t off = 0;
    L->hdr = off; off = align_up(off + sizeof(PlanHeader));
    L->tile_prefix = off; off = align_up(off + sizeof(int32_t) * (G + 1));
    L->part_offsets = off; off = align_up(off + sizeof(int32_t) * (G + 1));
    L->worker_group = off; off = align_up(off + sizeof(int32_t) * static_cast<size_t>(L->workers));
    L->q = off; off = align_up(off + sizeof(uint16_t) * G * d->num_heads * D);
    L->o_part = off; off = align_up(off + sizeof(float) * static_cast<size_t>(L->max_parts) * d->num_heads * d->kv_lora_rank);
    L->lse_part = off; off = align_up(off + sizeof(float) * static_cast<size_t>(L->max_parts) * d->num_heads);
    L->total = off;
    return MLA_OK;
}

template <typename K>
int ensure_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return MLA_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
        cudaSuccess) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

// ---- row GEMM plan ------------------------------------------------------
// tc: the tcgen05 row GEMM (N and the inner dimension multiples of 64): column
// tiles of 64 nb, the K-blocks of 64 split into `splits` ranges of
// k_per_split, one CTA per (column tile, row tile, range); the consumer sums
// the `splits` partials, four per memory round trip. The split is chosen to
// cover the weight in whole waves of CTAs (one per SM) at the least bytes per
// SM: weights, activations (from L2) and the partials' round trip, with the
// consumer's round trips counted as the bytes an SM streams in that time.
// Otherwise the CUDA-core GEMM writes `splits` partials.
struct AppendPlan {
    bool tc;
    int splits, k_per_split, nb;
};

AppendPlan append_plan(int32_t n_tokens, int32_t hidden, int32_t N) {
    AppendPlan a;
    a.tc = (N % 64 == 0) && (hidden % 64 == 0);
    a.nb = 1;
    if (a.tc) {
        const int64_t kb = hidden / 64, mt = (n_tokens + tc05::kRows - 1) / tc05::kRows, sms = num_sms();
        double best = -1.0;
        for (int nb = 4; nb >= 1; nb /= 2) {
            if (N % (64 * nb)) continue;
            const int64_t nt = N / (64 * nb);
            for (int64_t kpc = 1; kpc <= kb; ++kpc) {
                const int64_t z = (kb + kpc - 1) / kpc;
                if (kpc > 1 && (kb + kpc - 2) / (kpc - 1) == z) continue;  // a smaller kpc does the same
                const int64_t ctas = nt * mt * z, waves = (ctas + sms - 1) / sms;
                // bytes per SM: weights (HBM), activations (L2, a quarter of the cost), the
                // partials written and read back, and the consumer's memory round trips (one
                // per four partials, ~0.7 us, the bytes an SM streams meanwhile at ~44 GB/s)
                const double per_sm = static_cast<double>(waves) * kpc *
                                          (nb * 64.0 * tc05::kBoxBytes + 0.25 * tc05::kRows * tc05::kBoxBytes) +
                                      2.0 * 4.0 * z * n_tokens * N / sms + 31e3 * static_cast<double>((z + 3) / 4);
                if (best < 0 || per_sm < best) {
                    best = per_sm;
                    a.nb = nb;
                    a.k_per_split = static_cast<int>(kpc);
                    a.splits = static_cast<int>(z);
                }
            }
        }
        return a;
    }
    const int tile_n = kApTileN, tile_t = kApTileT, tile_k = kApTileK;
    const int64_t tiles = static_cast<int64_t>((N + tile_n - 1) / tile_n) * ((n_tokens + tile_t - 1) / tile_t);
    const int64_t target = 2 * num_sms();
    const int64_t chunks = (hidden + tile_k - 1) / tile_k;
    int64_t s = tiles >= target ? 1 : (target + tiles - 1) / tiles;
    if (s > chunks) s = chunks;
    if (s > 64) s = 64;
    if (s < 1) s = 1;
    const int64_t per = (chunks + s - 1) / s;  // K chunks per split
    a.k_per_split = static_cast<int>(per * tile_k);
    a.splits = static_cast<int>((chunks + per - 1) / per);
    return a;
}

// part[z][t][n] (fp32 [ap.splits][T][N]) = the K-range z of x . w on the
// tcgen05 row GEMM: x bf16 [T, K], w bf16 [K, N], K and N multiples of 64,
// x and w 16-byte aligned.
int launch_row_gemm(const void* x, int32_t T, int32_t K, const void* w, int32_t N, const AppendPlan& ap,
                    float* part, cudaStream_t st, const tc05::QHeadOut* qo = nullptr) {
    if (!aligned(x, 16) || !aligned(w, 16)) return MLA_ERR_INVALID_ARG;
    tc05::QHeadOut none{};
    if (!qo) qo = &none;
    CUtensorMap tm_x, tm_w;
    if (int rc = encode_2d(&tm_x, x, K, T, tc05::kRows)) return rc;
    if (int rc = encode_2d(&tm_w, w, N, K, 64)) return rc;
    const size_t smem = tc05::row_gemm_smem(ap.nb);
    if (int rc = ensure_smem(tc05::row_gemm_kernel, smem)) return rc;
    const dim3 grid(N / (64 * ap.nb), (T + tc05::kRows - 1) / tc05::kRows, ap.splits);
    return launch(tc05::row_gemm_kernel, grid, tc05::kThreads, smem, st, tm_x, tm_w, T, N, K / 64, ap.k_per_split,
                  ap.nb, part, *qo);
}

// The second product of the query projection writes q_nope / q_pe itself
// (tc05::QHeadOut) when every 64-column tile is one piece of one head.
bool q_heads_fused(const mla_dims_t* d) { return d->rope_dim == 64 && d->qk_nope_dim % 64 == 0; }

// ---- query projection workspace: GEMM 1 partials | c_q bf16 | GEMM 2 partials
struct QProjLayout {
    AppendPlan g1, g2;
    size_t part1, cq, part2, total;
};

int q_proj_layout(const mla_dims_t* d, int32_t T, int32_t hidden, int32_t R, QProjLayout* L) {
    if (int rc = check_dims(d)) return rc;
    if (T < 1 || hidden < 1 || R < 1) return MLA_ERR_INVALID_ARG;
    const int64_t N2 = static_cast<int64_t>(d->num_heads) * (d->qk_nope_dim + d->rope_dim);
    if (hidden % 64 || R % 64 || R > kQNormThreads * kQNormCols || N2 % 64 || N2 >= (int64_t(1) << 30) ||
        d->rope_dim % 2 ||
        d->rope_dim > 2 * kQMaxRopePairs || d->qk_nope_dim + d->rope_dim / 2 > 1024)
        return MLA_ERR_UNSUPPORTED_DIMS;
    L->g1 = append_plan(T, hidden, R);
    L->g2 = append_plan(T, R, static_cast<int32_t>(N2));
    if (q_heads_fused(d)) {
        // one K-range and the widest tile that divides N2: 256 columns per CTA stream
        // W_qb's rows in 512-byte pieces (measured 52 us against 64 for 64-column
        // tiles at 64 tokens on V3 dims)
        const int nb = N2 % 256 == 0 ? 4 : (N2 % 128 == 0 ? 2 : 1);
        L->g2 = AppendPlan{true, 1, R / 64, nb};
    }
    size_t off = 0;
    L->part1 = off; off = align_up(off + sizeof(float) * static_cast<size_t>(L->g1.splits) * T * R);
    L->cq = off; off = align_up(off + sizeof(uint16_t) * static_cast<size_t>(T) * R);
    L->part2 = off; off = align_up(off + sizeof(float) * static_cast<size_t>(L->g2.splits) * T * N2);
    L->total = off;
    return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int mla_version(void) { return 100; }

const char* mla_error_string(int s) {
    switch (s) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument";
        case MLA_ERR_UNSUPPORTED_DIMS: return "dims not supported by the selected kernel";
        case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MLA_ERR_CUDA: return "CUDA runtime or launch error";
        case MLA_ERR_DEVICE_FAULT: return "device fault: block id, slot or position out of range";
        case MLA_ERR_DEVICE_TIMEOUT: return "device timeout: a bounded wait expired";
        case MLA_ERR_NO_DEVICE: return "no sm_100 CUDA device is current";
        case MLA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the fixed no-allocation buffer";
        default: return "unknown status";
    }
}

int mla_get_device_error(int* device_status, void* stream) {
    if (!device_status) return MLA_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MLA_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
    *device_status = v;
    return MLA_OK;
}

size_t mla_append_workspace_size(const mla_dims_t* dims, int32_t n_tokens, int32_t hidden) {
    if (check_dims(dims) || n_tokens < 1 || hidden < 1) return 0;
    const int N = dims->kv_lora_rank + dims->rope_dim;
    const AppendPlan a = append_plan(n_tokens, hidden, N);
    return align_up(sizeof(float) * static_cast<size_t>(a.splits) * n_tokens * N);
}

static int append_kv(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden, const void* w_kva,
                     const void* rms_gamma, float rms_eps, float rope_base, const int32_t* seq_ids,
                     const int32_t* positions, const int32_t* block_table, int32_t num_seqs,
                     int32_t max_blocks_per_seq, void* pool, int64_t num_blocks, void* workspace,
                     size_t workspace_bytes, void* stream, bool fp8_cache) {
    if (int rc = check_dims(dims)) return rc;
    if (fp8_cache && !fp8_dims_ok(dims)) return MLA_ERR_UNSUPPORTED_DIMS;
    if (!x || !w_kva || !seq_ids || !positions || !block_table || !pool || !workspace) return MLA_ERR_INVALID_ARG;
    if (n_tokens < 1 || hidden < 1 || num_seqs < 1 || max_blocks_per_seq < 1 || num_blocks < 1)
        return MLA_ERR_INVALID_ARG;
    if (!(rms_eps >= 0.f) || !(rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign) || !aligned(pool, 16)) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_append_workspace_size(dims, n_tokens, hidden)) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (dims->kv_lora_rank + dims->rope_dim > 1024) return MLA_ERR_UNSUPPORTED_DIMS;  // epilogue: 4 columns per thread
    if (int rc = device_ok()) return rc;
    const int N = dims->kv_lora_rank + dims->rope_dim;
    const AppendPlan ap = append_plan(n_tokens, hidden, N);
    const int splits = ap.splits;  // partials the epilogue sums
    float* part = static_cast<float*>(workspace);
    cudaStream_t st = as_stream(stream);
    if (ap.tc) {
        if (int rc = launch_row_gemm(x, n_tokens, hidden, w_kva, N, ap, part, st)) return rc;
    } else {
        dim3 g1((N + kApTileN - 1) / kApTileN, (n_tokens + kApTileT - 1) / kApTileT, splits);
        if (int rc = launch(append_gemm_kernel, g1, 256, 0, st, static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w_kva),
                                               part, n_tokens, hidden, N, ap.k_per_split)) return rc;
    }
    if (int rc = launch_status()) return rc;
    AppendEpilogueParams P;
    P.part = part;
    P.gamma = static_cast<const uint16_t*>(rms_gamma);
    P.seq_ids = seq_ids;
    P.positions = positions;
    P.block_table = block_table;
    P.pool = static_cast<uint16_t*>(pool);
    P.pool8 = static_cast<uint8_t*>(pool);
    P.layout8 = fp8::Layout{fp8::row_bytes(dims->kv_lora_rank, dims->rope_dim),
                            fp8::block_bytes(dims->kv_lora_rank, dims->rope_dim, dims->block_size), dims->block_size};
    P.fp8 = fp8_cache ? 1 : 0;
    P.num_blocks = num_blocks;
    P.splits = splits;
    P.T = n_tokens;
    P.dc = dims->kv_lora_rank;
    P.dr = dims->rope_dim;
    P.num_seqs = num_seqs;
    P.max_blocks_per_seq = max_blocks_per_seq;
    P.block_size = dims->block_size;
    P.eps = rms_eps;
    P.rope_base = rope_base;
    if (int rc = launch(append_epilogue_kernel, n_tokens, 256, sizeof(float) * N, st, P)) return rc;
    return launch_status();
}

int mla_append_kv(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden, const void* w_kva,
                  const void* rms_gamma, float rms_eps, float rope_base, const int32_t* seq_ids,
                  const int32_t* positions, const int32_t* block_table, int32_t num_seqs,
                  int32_t max_blocks_per_seq, void* pool, int64_t num_blocks, void* workspace,
                  size_t workspace_bytes, void* stream) {
    return append_kv(dims, x, n_tokens, hidden, w_kva, rms_gamma, rms_eps, rope_base, seq_ids, positions,
                     block_table, num_seqs, max_blocks_per_seq, pool, num_blocks, workspace, workspace_bytes, stream,
                     false);
}

int mla_append_kv_fp8(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden, const void* w_kva,
                      const void* rms_gamma, float rms_eps, float rope_base, const int32_t* seq_ids,
                      const int32_t* positions, const int32_t* block_table, int32_t num_seqs,
                      int32_t max_blocks_per_seq, void* pool_fp8, int64_t num_blocks, void* workspace,
                      size_t workspace_bytes, void* stream) {
    return append_kv(dims, x, n_tokens, hidden, w_kva, rms_gamma, rms_eps, rope_base, seq_ids, positions,
                     block_table, num_seqs, max_blocks_per_seq, pool_fp8, num_blocks, workspace, workspace_bytes,
                     stream, true);
}

size_t mla_fp8_block_bytes(const mla_dims_t* dims) {
    if (check_dims(dims) || !fp8_dims_ok(dims)) return 0;
    return static_cast<size_t>(fp8::block_bytes(dims->kv_lora_rank, dims->rope_dim, dims->block_size));
}

int mla_cache_to_fp8(const mla_dims_t* dims, const void* pool, int64_t num_blocks, void* pool_fp8, void* stream) {
    if (int rc = check_dims(dims)) return rc;
    if (!fp8_dims_ok(dims)) return MLA_ERR_UNSUPPORTED_DIMS;
    if (!pool || !pool_fp8 || num_blocks < 1) return MLA_ERR_INVALID_ARG;
    if (!aligned(pool, 16) || !aligned(pool_fp8, 16)) return MLA_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    const int64_t rows = num_blocks * dims->block_size;
    const fp8::Layout L{fp8::row_bytes(dims->kv_lora_rank, dims->rope_dim),
                        fp8::block_bytes(dims->kv_lora_rank, dims->rope_dim, dims->block_size), dims->block_size};
    const int64_t grid = (rows + 7) / 8;
    if (grid > 0x7FFFFFFF) return MLA_ERR_INVALID_ARG;
    if (int rc = launch(fp8::quantize_pool_kernel, static_cast<unsigned>(grid), 256, 0, as_stream(stream),
                        static_cast<const uint16_t*>(pool), rows, dims->kv_lora_rank, dims->rope_dim, L,
                        static_cast<uint8_t*>(pool_fp8)))
        return rc;
    return launch_status();
}

size_t mla_q_proj_workspace_size(const mla_dims_t* dims, int32_t n_tokens, int32_t hidden, int32_t q_rank) {
    QProjLayout L;
    return q_proj_layout(dims, n_tokens, hidden, q_rank, &L) ? 0 : L.total;
}

int mla_q_proj(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden, const void* w_qa,
               int32_t q_rank, const void* q_gamma, float rms_eps, const void* w_qb, const int32_t* positions,
               float rope_base, void* q_nope, void* q_pe, void* workspace, size_t workspace_bytes, void* stream) {
    QProjLayout L;
    if (int rc = q_proj_layout(dims, n_tokens, hidden, q_rank, &L)) return rc;
    if (!x || !w_qa || !w_qb || !positions || !q_nope || !q_pe || !workspace) return MLA_ERR_INVALID_ARG;
    if (!(rms_eps >= 0.f) || !(rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign)) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (int rc = device_ok()) return rc;
    cudaStream_t st = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* part1 = reinterpret_cast<float*>(ws + L.part1);
    uint16_t* cq = reinterpret_cast<uint16_t*>(ws + L.cq);
    float* part2 = reinterpret_cast<float*>(ws + L.part2);
    const int32_t H = dims->num_heads, dn = dims->qk_nope_dim, dr = dims->rope_dim;
    const int32_t N2 = H * (dn + dr);
    // c_q = RMSNorm(x . W_qa) * gamma, rounded to bf16 as the second GEMM's operand
    if (int rc = launch_row_gemm(x, n_tokens, hidden, w_qa, q_rank, L.g1, part1, st)) return rc;
    if (int rc = launch(q_norm_kernel, n_tokens, kQNormThreads, sizeof(float) * q_rank, st, part1, L.g1.splits,
                        n_tokens, q_rank, static_cast<const uint16_t*>(q_gamma), rms_eps, cq)) return rc;
    // q = c_q . W_qb, then the per-head split and the RoPE of the rope part
    if (q_heads_fused(dims)) {
        if (!aligned(q_nope, 16) || !aligned(q_pe, 16)) return MLA_ERR_INVALID_ARG;
        tc05::QHeadOut qo;
        qo.positions = positions;
        qo.q_nope = static_cast<uint16_t*>(q_nope);
        qo.q_pe = static_cast<uint16_t*>(q_pe);
        qo.dn = dn;
        for (int i = 0; i < 32; ++i) qo.inv_freq[i] = std::pow(static_cast<double>(rope_base), -2.0 * i / 64.0);
        if (int rc = launch_row_gemm(cq, n_tokens, q_rank, w_qb, N2, L.g2, part2, st, &qo)) return rc;
        return launch_status();
    }
    if (int rc = launch_row_gemm(cq, n_tokens, q_rank, w_qb, N2, L.g2, part2, st)) return rc;
    QSplitParams P;
    P.part = part2;
    P.positions = positions;
    P.q_nope = static_cast<uint16_t*>(q_nope);
    P.q_pe = static_cast<uint16_t*>(q_pe);
    P.splits = L.g2.splits;
    P.T = n_tokens;
    P.H = H;
    P.dn = dn;
    P.dr = dr;
    for (int i = 0; i < kQMaxRopePairs; ++i)
        P.inv_freq[i] = i < dr / 2 ? std::pow(static_cast<double>(rope_base), -2.0 * i / static_cast<double>(dr)) : 0.0;
    const int threads = (dn + dr / 2 + 31) / 32 * 32;
    if (int rc = launch(q_split_rope_kernel, dim3(n_tokens, H), threads, 0, st, P)) return rc;
    return launch_status();
}

size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t batch, int32_t q_len, int32_t max_context_len,
                                 const mla_decode_opts_t* opts) {
    DecodeLayout L;
    if (decode_layout(dims, batch, q_len, max_context_len, opts, &L)) return 0;
    return L.total;
}

// Timing hook: inside a stream capture the event becomes an external
// event-record node of the graph, so that it is recorded on every replay.
static void record_hook(void* ev, cudaStream_t st) {
    if (!ev) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), st, cudaEventRecordExternal);
    else
        cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

// The attention launch waits for the caller's cache-ready event, if any.
static int wait_hook(void* ev, cudaStream_t st) {
    if (!ev) return MLA_OK;
    return cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(ev), 0) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode(const mla_dims_t* dims, const void* q_nope, const void* q_pe, int32_t batch, int32_t q_len,
               const void* pool, int64_t num_blocks, const int32_t* block_table, int32_t max_blocks_per_seq,
               const int32_t* context_lens, int32_t max_context_len, const void* w_uk, const void* w_uv,
               void* out, void* workspace, size_t workspace_bytes, const mla_decode_opts_t* opts, void* stream) {
    DecodeLayout L;
    if (int rc = decode_layout(dims, batch, q_len, max_context_len, opts, &L)) return rc;
    if (!q_nope || !q_pe || !pool || !block_table || !context_lens || !w_uk || !w_uv || !out || !workspace)
        return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || max_blocks_per_seq < 1) return MLA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(max_blocks_per_seq) * dims->block_size < max_context_len) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign) || !aligned(pool, 16)) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (int rc = device_ok()) return rc;

    cudaStream_t st = as_stream(stream);
    char* ws = static_cast<char*>(workspace);
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(ws + L.hdr);
    int32_t* tile_prefix = reinterpret_cast<int32_t*>(ws + L.tile_prefix);
    int32_t* part_offsets = reinterpret_cast<int32_t*>(ws + L.part_offsets);
    int32_t* worker_group = reinterpret_cast<int32_t*>(ws + L.worker_group);
    uint16_t* q = reinterpret_cast<uint16_t*>(ws + L.q);
    float* o_part = reinterpret_cast<float*>(ws + L.o_part);
    float* lse_part = reinterpret_cast<float*>(ws + L.lse_part);
    const int32_t G = batch * q_len;
    const int H = dims->num_heads, dc = dims->kv_lora_rank, dr = dims->rope_dim;

    // The tcgen05 absorption, merge and up-projection kernels take their
    // operands through TMA (16-byte aligned); other dims or alignments use the
    // CUDA-core kernels. The tensor-core attention writes bf16 partials, which
    // only the tcgen05 merge reads, so it needs the tcgen05 kernels around it.
    const bool tc05 = tc05_dims_ok(dims) && aligned(q_nope, 16) && aligned(q_pe, 16) && aligned(w_uk, 16) &&
                      aligned(w_uv, 16) && aligned(out, 16);
    if (L.kernel == kKernelPair && !tc05) return MLA_ERR_INVALID_ARG;
    const bool fp8_cache = opts && opts->cache_fp8;  // decode_layout admits it with the tcgen05 kernel only
    const bool latent_out = opts && opts->output_latent;
    if (latent_out && !tc05) return MLA_ERR_UNSUPPORTED_DIMS;  // o_lat comes from the tensor-core merge

    const size_t plan_smem = sizeof(int32_t) * (static_cast<size_t>(G) + 1);
    const int32_t prefix_in_smem = plan_smem <= 48 * 1024 ? 1 : 0;
    if (int rc = launch(plan_kernel, 1, 1024, prefix_in_smem ? plan_smem : 0, st, context_lens, batch, q_len, L.tile,
                        L.workers, hdr, tile_prefix, part_offsets, worker_group, prefix_in_smem)) return rc;
    if (int rc = launch_status()) return rc;

    if (tc05) {
        CUtensorMap tm_qn, tm_wuk;
        if (int rc = encode_2d(&tm_qn, q_nope, static_cast<uint64_t>(H) * dims->qk_nope_dim, G, tc05::kRows)) return rc;
        if (int rc = encode_2d(&tm_wuk, w_uk, dc, static_cast<uint64_t>(H) * dims->qk_nope_dim, dims->qk_nope_dim))
            return rc;
        const size_t smem = tc05::absorb_smem(dims->qk_nope_dim);
        if (int rc = ensure_smem(tc05::absorb_kernel, smem)) return rc;
        if (int rc = launch(tc05::absorb_kernel, dim3(H, (G + tc05::kRows - 1) / tc05::kRows, dc / 256), tc05::kThreads, smem, st,
            tm_qn, tm_wuk, static_cast<const uint16_t*>(q_pe), G, H, dims->qk_nope_dim, dc, dr, q,
            fp8_cache ? 1 : 0)) return rc;
    } else {
        const size_t absorb_smem = sizeof(float) * kAbsorbGroups * dims->qk_nope_dim;
        if (int rc = ensure_smem(absorb_q_kernel, absorb_smem)) return rc;
        if (int rc = launch(absorb_q_kernel, dim3(H, (G + kAbsorbGroups - 1) / kAbsorbGroups), kAbsorbThreads, absorb_smem, st,
            static_cast<const uint16_t*>(q_nope), static_cast<const uint16_t*>(q_pe),
            static_cast<const uint16_t*>(w_uk), q, G, H, dims->qk_nope_dim, dc, dr)) return rc;
    }
    if (int rc = launch_status()) return rc;

    if (L.kernel == kKernelPair) {
        CUtensorMap tm_q, tm_k3, tm_k2, tm_v;
        F8Maps f8;
        const uint64_t pool_rows = static_cast<uint64_t>(num_blocks) * dims->block_size;
        if (int rc = encode_row_blocks(&tm_q, q, pair::kD, static_cast<uint64_t>(G) * H, 64, pair::kQBoxes)) return rc;
        if (fp8_cache) {
            if (int rc = encode_f8_maps(&f8, pool, dims, num_blocks)) return rc;
        } else {
            if (int rc = encode_row_blocks(&tm_k3, pool, pair::kD, pool_rows, 64, 3)) return rc;
            if (int rc = encode_row_blocks(&tm_k2, pool, pair::kD, pool_rows, 64, 2)) return rc;
            if (int rc = encode_row_blocks(&tm_v, pool, pair::kD, pool_rows, 32, 4)) return rc;
        }
        pair::Params PP;
        PP.hdr = hdr;
        PP.worker_group = worker_group;
        PP.tile_prefix = tile_prefix;
        PP.part_offsets = part_offsets;
        PP.context_lens = context_lens;
        PP.block_table = block_table;
        PP.pool = static_cast<const uint8_t*>(pool);
        PP.o_part = reinterpret_cast<uint16_t*>(o_part);  // bf16 partials (the slot layout keeps fp32 size)
        PP.lse_part = lse_part;
        PP.num_blocks = num_blocks;
        PP.batch = batch;
        PP.max_blocks_per_seq = max_blocks_per_seq;
        PP.block_size = dims->block_size;
        PP.q_len = q_len;
        PP.scale_log2 = dims->softmax_scale * 1.4426950408889634f;
        PP.wait_ns = (opts && opts->debug_wait_limit_us) ? 1000ull * opts->debug_wait_limit_us : ptx::kWaitLimitNs;
        PP.starve = (opts && opts->debug_starve) ? 1 : 0;
        PP.f8_block_bytes = fp8::block_bytes(dc, dr, dims->block_size);
        if (int rc = ensure_smem(pair::pair_decode_kernel, pair::kSmemBytes)) return rc;
        if (int rc = ensure_smem(pair::pair_decode_f8_kernel, pair::kSmemBytes)) return rc;
        if (int rc = wait_hook(opts ? opts->cache_ready : nullptr, st)) return rc;
        record_hook(opts ? opts->event_attn_begin : nullptr, st);
        if (fp8_cache) {
            if (int rc = launch(pair::pair_decode_f8_kernel, 2 * L.workers, pair::kF8Threads, pair::kSmemBytes, st,
                                tm_q, f8.k8, f8.ks, f8.kr, f8.v8, f8.vs, PP)) return rc;
        } else {
            if (int rc = launch(pair::pair_decode_kernel, 2 * L.workers, pair::kThreads, pair::kSmemBytes, st, tm_q,
                                tm_k3, tm_k2, tm_v, PP)) return rc;
        }
        if (int rc = launch_status()) return rc;
        record_hook(opts ? opts->event_attn_end : nullptr, st);
    } else {
    GenericDecodeParams P;
    P.q = q;
    P.pool = static_cast<const uint16_t*>(pool);
    P.block_table = block_table;
    P.context_lens = context_lens;
    P.hdr = hdr;
    P.worker_group = worker_group;
    P.tile_prefix = tile_prefix;
    P.part_offsets = part_offsets;
    P.o_part = o_part;
    P.lse_part = lse_part;
    P.num_blocks = num_blocks;
    P.batch = batch;
    P.max_blocks_per_seq = max_blocks_per_seq;
    P.block_size = dims->block_size;
    P.q_len = q_len;
    P.H = H;
    P.dc = dc;
    P.dr = dr;
    P.scale = dims->softmax_scale;
    const size_t gsmem = generic_decode_smem(dc, dr);
    if (int rc = ensure_smem(generic_decode_kernel, gsmem)) return rc;
    if (int rc = wait_hook(opts ? opts->cache_ready : nullptr, st)) return rc;
    record_hook(opts ? opts->event_attn_begin : nullptr, st);
    if (int rc = launch(generic_decode_kernel, dim3(L.workers, (H + kGenHeads - 1) / kGenHeads), kGenThreads, gsmem, st, P)) return rc;
    if (int rc = launch_status()) return rc;
    record_hook(opts ? opts->event_attn_end : nullptr, st);
    }

    // the fused merge + up-projection takes bf16 partials, d_v = 128 and at most
    // 64 * kMuvMaxBox partial slots per block of 64 groups (<= 64 + workers - 1)
    const int muv_box = static_cast<int>((std::min<int64_t>(G, tc05::kMuvRows) + L.workers - 1 + 63) / 64);
    if (latent_out) {
        // out = o_lat (bf16 [G, H, d_c]): the merge only; W_UV is applied later, absorbed into W_O
        uint16_t* o_lat = static_cast<uint16_t*>(out);
        const dim3 mgrid(G, (H + 3) / 4);
        if (L.kernel == kKernelPair) {
            if (int rc = launch(tc05::merge_kernel<uint16_t>, mgrid, 128, 0, st,
                                reinterpret_cast<const uint16_t*>(o_part), lse_part, part_offsets, G, H, dc, o_lat))
                return rc;
        } else {
            if (int rc = launch(tc05::merge_kernel<float>, mgrid, 128, 0, st, o_part, lse_part, part_offsets, G, H, dc,
                                o_lat))
                return rc;
        }
    } else if (tc05 && L.kernel == kKernelPair && dims->v_head_dim == tc05::kMuvDv && muv_box <= tc05::kMuvMaxBox) {
        CUtensorMap tm_wuv, tm_p;
        if (int rc = encode_2d(&tm_wuv, w_uv, dc, static_cast<uint64_t>(H) * tc05::kMuvDv, tc05::kMuvDv)) return rc;
        if (int rc = encode_parts(&tm_p, o_part, dc, H, L.max_parts)) return rc;
        const size_t smem = tc05::merge_uv_smem(muv_box);
        if (int rc = ensure_smem(tc05::merge_uv_kernel, smem)) return rc;
        if (int rc = launch(tc05::merge_uv_kernel, dim3(H, (G + tc05::kMuvRows - 1) / tc05::kMuvRows),
                            tc05::kMuvThreads, smem, st, tm_wuv, tm_p, lse_part, part_offsets, G, H, dc, muv_box,
                            static_cast<uint16_t*>(out)))
            return rc;
    } else if (tc05) {
        // merge into bf16 o_lat (the absorbed queries are dead once the attention is done:
        // o_lat reuses their space), then the up-projection
        uint16_t* o_lat = q;
        const dim3 mgrid(G, (H + 3) / 4);
        if (L.kernel == kKernelPair) {
            if (int rc = launch(tc05::merge_kernel<uint16_t>, mgrid, 128, 0, st,
                                reinterpret_cast<const uint16_t*>(o_part), lse_part, part_offsets, G, H, dc, o_lat))
                return rc;
        } else {
            if (int rc = launch(tc05::merge_kernel<float>, mgrid, 128, 0, st, o_part, lse_part, part_offsets, G, H, dc,
                                o_lat))
                return rc;
        }
        if (int rc = launch_status()) return rc;
        CUtensorMap tm_ol, tm_wuv;
        if (int rc = encode_2d(&tm_ol, o_lat, static_cast<uint64_t>(H) * dc, G, tc05::kRows)) return rc;
        if (int rc = encode_2d(&tm_wuv, w_uv, dc, static_cast<uint64_t>(H) * dims->v_head_dim, dims->v_head_dim))
            return rc;
        const size_t smem = tc05::uv_smem(dims->v_head_dim);
        if (int rc = ensure_smem(tc05::uv_kernel, smem)) return rc;
        if (int rc = launch(tc05::uv_kernel, dim3(H, (G + tc05::kRows - 1) / tc05::kRows), tc05::kThreads, smem, st,
            tm_ol, tm_wuv, G, H, dc, dims->v_head_dim, static_cast<uint16_t*>(out))) return rc;
    } else {
        const size_t uv_smem = sizeof(float) * kUvGroups * dc;
        if (int rc = ensure_smem(combine_uv_kernel, uv_smem)) return rc;
        if (int rc = launch(combine_uv_kernel, dim3(H, (G + kUvGroups - 1) / kUvGroups), kUvThreads, uv_smem, st,
            o_part, lse_part, part_offsets, static_cast<const uint16_t*>(w_uv), G, H, dc, dims->v_head_dim,
            static_cast<uint16_t*>(out))) return rc;
    }
    return launch_status();
}

size_t mla_o_proj_workspace_size(int32_t n_tokens, int32_t k, int32_t n) {
    if (n_tokens < 1 || k < 64 || n < 64 || k % 64 || n % 64) return 0;
    const AppendPlan a = append_plan(n_tokens, k, n);
    return align_up(sizeof(float) * static_cast<size_t>(a.splits) * n_tokens * n);
}

int mla_o_proj(const void* x, int32_t n_tokens, int32_t k, const void* w, int32_t n, void* y, void* workspace,
               size_t workspace_bytes, void* stream) {
    if (!x || !w || !y || !workspace || n_tokens < 1 || k < 1 || n < 1) return MLA_ERR_INVALID_ARG;
    if (k % 64 || n % 64) return MLA_ERR_UNSUPPORTED_DIMS;
    if (!aligned(workspace, kAlign) || !aligned(x, 16) || !aligned(w, 16) || !aligned(y, 8)) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_o_proj_workspace_size(n_tokens, k, n)) return MLA_ERR_WORKSPACE_TOO_SMALL;
    if (int rc = device_ok()) return rc;
    cudaStream_t st = as_stream(stream);
    const AppendPlan ap = append_plan(n_tokens, k, n);
    float* part = static_cast<float*>(workspace);
    if (int rc = launch_row_gemm(x, n_tokens, k, w, n, ap, part, st)) return rc;
    const int64_t quads = static_cast<int64_t>(n_tokens) * n / 4;
    if (int rc = launch(tc05::sum_partials_kernel, static_cast<unsigned>((quads + 127) / 128), 128, 0, st,
                        static_cast<const float*>(part), ap.splits, n_tokens, n, static_cast<uint16_t*>(y)))
        return rc;
    return launch_status();
}

int mla_combine(const mla_dims_t* dims, const float* o_part, const float* lse_part, const int32_t* part_offsets,
                int32_t n_groups, float* o_lat, float* lse_out, void* stream) {
    if (int rc = check_dims(dims)) return rc;
    if (!o_part || !lse_part || !part_offsets || !o_lat || n_groups < 1) return MLA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(n_groups) * dims->num_heads >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED_DIMS;
    if (int rc = device_ok()) return rc;
    if (int rc = launch(combine_kernel, n_groups * dims->num_heads, 128, 0, as_stream(stream),
        o_part, lse_part, part_offsets, n_groups, dims->num_heads, dims->kv_lora_rank, o_lat, lse_out)) return rc;
    return launch_status();
}

int mla_debug_resolve_slots(const mla_dims_t* dims, const int32_t* block_table, int32_t num_seqs,
                            int32_t max_blocks_per_seq, int64_t num_blocks, const int32_t* seq_ids,
                            const int32_t* positions, int32_t n, int64_t* rows, void* stream) {
    if (int rc = check_dims(dims)) return rc;
    if (!block_table || !seq_ids || !positions || !rows || n < 1 || num_seqs < 1 || max_blocks_per_seq < 1)
        return MLA_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    if (int rc = launch(resolve_slots_kernel, (n + 255) / 256, 256, 0, as_stream(stream),
        block_table, num_seqs, max_blocks_per_seq, num_blocks, dims->block_size, seq_ids, positions, n, rows)) return rc;
    return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without allocation: the scratch comes from a buffer compiled into
// the library instead of a caller-provided workspace. It exists for callers
// that cannot allocate device memory themselves (see mla_b200.h). Host code
// must not pass `g_no_alloc_scratch` itself to a kernel: on the host that
// name is only a stand-in for the symbol. The device address is looked up
// with cudaGetSymbolAddress once per CUDA context, with that context current,
// and cached under the context's process-unique id (cuCtxGetId), so that a
// context created later (another device, a driver-API context, the primary
// context re-created after cudaDeviceReset) never sees a stale address.
namespace mla {
namespace {

static __device__ __align__(256) unsigned char g_no_alloc_scratch[MLA_NO_ALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return reinterpret_cast<F>(p);
}

// Process-unique id of the current context; false if none is current.
bool current_context_id(unsigned long long* id) {
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchEntry {
    unsigned long long ctx_id;
    void* ptr;
};
std::mutex g_no_alloc_mutex;
ScratchEntry g_no_alloc_cache[64] = {};
int g_no_alloc_next = 0;

int no_alloc_scratch(void** out) {
    std::lock_guard<std::mutex> lock(g_no_alloc_mutex);
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (have_id)
        for (const ScratchEntry& e : g_no_alloc_cache)
            if (e.ptr && e.ctx_id == id) {
                *out = e.ptr;
                return MLA_OK;
            }
    void* p = nullptr;  // first call in this context (the look-up makes the runtime's context current)
    if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    if (have_id || current_context_id(&id)) {
        g_no_alloc_cache[g_no_alloc_next] = ScratchEntry{id, p};
        g_no_alloc_next = (g_no_alloc_next + 1) % 64;
    }
    *out = p;
    return MLA_OK;
}

}  // namespace
}  // namespace mla

extern "C" int mla_decode_no_alloc(const mla_dims_t* dims, const void* q_nope, const void* q_pe, int32_t batch,
                                   int32_t q_len, const void* pool, int64_t num_blocks, const int32_t* block_table,
                                   int32_t max_blocks_per_seq, const int32_t* context_lens,
                                   int32_t max_context_len, const void* w_uk, const void* w_uv, void* out,
                                   const mla_decode_opts_t* opts, void* stream) {
    const size_t need = mla_decode_workspace_size(dims, batch, q_len, max_context_len, opts);
    if (need == 0) {  // the same validation result as mla_decode
        DecodeLayout L;
        const int rc = decode_layout(dims, batch, q_len, max_context_len, opts, &L);
        return rc ? rc : MLA_ERR_INVALID_ARG;
    }
    if (need > MLA_NO_ALLOC_SCRATCH_BYTES) return MLA_ERR_SCRATCH_LIMIT;
    if (int rc = device_ok()) return rc;
    void* scratch = nullptr;
    if (int rc = no_alloc_scratch(&scratch)) return rc;
    return mla_decode(dims, q_nope, q_pe, batch, q_len, pool, num_blocks, block_table, max_blocks_per_seq,
                      context_lens, max_context_len, w_uk, w_uv, out, scratch, MLA_NO_ALLOC_SCRATCH_BYTES, opts,
                      stream);
}
