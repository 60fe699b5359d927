/*
 * mla_b200.h -- C ABI of the B200 (sm_100a) MLA absorbed-decode library.
 *
 * Multi-head Latent Attention (DeepSeek-V3 style) keeps one latent row per
 * cached token: c_kv (kv_lora_rank values, RMS-normalised) followed by a
 * decoupled RoPE key k_pe (rope_dim values) shared by every head.
 * Sources, cited by page title and section:
 *   [MLA-arch] "MLA架构：低秩注意力机制优化LLM显存与计算效率": section 1
 *              (128 heads, qk_head_dim 128 + 64, the RoPE part broadcast to
 *              all heads), 2.2 (kv_a_proj_with_mqa hidden -> 512 + 64,
 *              kv_a_layernorm, kv_b_proj), 3.1 (absorption = matrix
 *              associativity), 3.2 (cache = c_kv + shared pe), 4.2 (fuse
 *              RoPE with the cache update).
 *   [MQA-MLA]  "一次讲透MHA、GQA、MQA、MLA", section "MLA的实现": RoPE module,
 *              forward_training (explicit K/V) and forward_inference_absorbed
 *              (scores = q_absorbed . c_kv + q_r . k_r; output from P . c_kv).
 *
 * Conventions for every entry point:
 *   - bf16 means IEEE bfloat16 stored as uint16; all tensors are dense,
 *     row-major, with the shapes given below.
 *   - Pointers are DEVICE pointers unless the argument says "host". The
 *     caller allocates and owns every buffer; the library never allocates,
 *     frees or synchronises. Work is enqueued on `stream` (a cudaStream_t;
 *     NULL = legacy default stream) and runs asynchronously.
 *   - Return value: MLA_OK (0) or a negative mla_status_t. Host-side
 *     validation failures return before anything is enqueued. Nothing
 *     aborts, throws or prints across this boundary.
 *   - Faults found by a kernel (a block id outside the pool, a position
 *     outside the block table, a bounded device wait that expired) do not
 *     trap: the offending access is skipped and a device error word is set;
 *     read and clear it with mla_get_device_error().
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = -1,         /* null pointer, non-positive size, bad stride */
    MLA_ERR_UNSUPPORTED_DIMS = -2,    /* dims outside what the kernels implement */
    MLA_ERR_WORKSPACE_TOO_SMALL = -3, /* workspace_bytes < the *_workspace_size() answer */
    MLA_ERR_CUDA = -4,                /* a CUDA runtime call or launch failed */
    MLA_ERR_DEVICE_FAULT = -5,        /* device error word: bad block id / slot / position */
    MLA_ERR_DEVICE_TIMEOUT = -6,      /* device error word: a bounded wait expired */
    MLA_ERR_NO_DEVICE = -7,           /* no sm_100 device is current */
    MLA_ERR_SCRATCH_LIMIT = -8        /* mla_decode_no_alloc: the problem needs more
                                         scratch than MLA_NO_ALLOC_SCRATCH_BYTES */
} mla_status_t;

/* Per-layer sizes. DeepSeek-V3: {128, 512, 64, 128, 128, 64, 1/sqrt(192)}
 * ([MLA-arch] 1 and 2.2). softmax_scale multiplies the summed score
 * q_nope.k_nope + q_pe.k_pe; the pages use (d_nope + d_rope)^-1/2
 * ([MQA-MLA] "MLA的实现", self.scale). */
typedef struct mla_dims {
    int32_t num_heads;    /* H */
    int32_t kv_lora_rank; /* d_c: latent values per token */
    int32_t rope_dim;     /* d_r: shared RoPE key values per token */
    int32_t qk_nope_dim;  /* d_n: per-head query/key width without RoPE */
    int32_t v_head_dim;   /* d_v: per-head value width */
    int32_t block_size;   /* tokens per cache page */
    float softmax_scale;
} mla_dims_t;

/* Kernel choice, split control and timing hooks for mla_decode. Pass NULL
 * for defaults. */
typedef struct mla_decode_opts {
    int32_t kernel;      /* 0 auto; 1 sm100 tensor-core kernel (V3 dims only);
                            2 CUDA-core kernel (any supported dims) */
    int32_t num_workers; /* 0 auto (tensor-core kernel: one worker per SM
                            pair, but at most half of the problem's 128-token
                            tiles, batch * q_len * ceil(max_context_len / 128),
                            so that a small problem keeps about two tiles per
                            worker); else the number of split-KV workers the
                            balanced schedule targets (>= 1) */
    void* event_attn_begin; /* NULL or a cudaEvent_t recorded on `stream` right
                               before the split-KV attention kernel */
    void* event_attn_end;   /* NULL or a cudaEvent_t recorded right after it.
                               Under stream capture both are captured as
                               external event-record nodes, so a graph
                               replay records them again. */
    void* cache_ready;      /* NULL or a cudaEvent_t that the attention
                               launch (the first launch that reads the
                               cache) waits for (cudaStreamWaitEvent on
                               `stream`). Record it after an mla_append_kv
                               issued on another stream: the append then
                               runs beside the schedule and the query
                               absorption, which do not read the cache.
                               Under stream capture it joins the two
                               streams' work into one graph. */
    /* Test hooks of the failure detection, 0 in normal use. Every wait of
     * the tensor-core attention kernel (an mbarrier that a copy, a
     * tensor-core operation or another warp completes) gives up after a
     * time limit, records MLA_ERR_DEVICE_TIMEOUT in the device error word
     * and lets the kernel drain and exit, so that the context stays usable.
     * debug_wait_limit_us replaces the default limit of 2 s (0 = default).
     * debug_starve != 0 makes that kernel's load warps issue nothing, so that
     * no copy or tensor-core operation is ever in flight and every consumer
     * wait runs out; the call then reports MLA_ERR_DEVICE_TIMEOUT through
     * mla_get_device_error() and its output is undefined. */
    uint32_t debug_wait_limit_us;
    int32_t debug_starve;
    /* 0: out = W_UV o_lat per head (bf16 [batch, q_len, H, v_head_dim]).
     * 1: out receives o_lat itself (bf16 [batch, q_len, H, kv_lora_rank]) and
     * w_uv is not read: the input of the full absorption of W_UV into the
     * output projection ([MQA-MLA] "MLA的实现", forward_inference_absorbed,
     * W_o_absorbed = W_UV^T W_O; [MLA-arch] 3.1), applied with mla_o_proj.
     * Needs the tensor-core merge (kv_lora_rank 256 or 512, the alignment
     * below), else MLA_ERR_UNSUPPORTED_DIMS before anything is enqueued. */
    int32_t output_latent;
    /* 0: `pool` is the bf16 cache. 1: `pool` is the FP8 cache (layout below;
     * num_blocks blocks of mla_fp8_block_bytes()). The tensor-core kernel
     * reads it (DeepSeek-V3 dims); anything else returns
     * MLA_ERR_UNSUPPORTED_DIMS before enqueuing. */
    int32_t cache_fp8;
} mla_decode_opts_t;

/* Paged latent cache ("pool"), [MLA-arch] 3.2 kept as one row per token:
 *   pool        bf16 [num_blocks, block_size, kv_lora_rank + rope_dim]
 *               row = c_kv (kv_lora_rank) then k_pe (rope_dim)
 *   block_table int32 [batch, max_blocks_per_seq]; page j of sequence b is
 *               pool block block_table[b*max_blocks_per_seq + j]
 *   token t of sequence b lives in pool row
 *               block_table[b][t / block_size] * block_size + t % block_size
 * A contiguous cache is block_size >= context length with block b for
 * sequence b. */

/* FP8 latent cache. [MLA-arch] 4.2 item 3 ("量化的影响") notes that
 * quantising the cache shrinks it further and warns about numerical
 * stability; it fixes no format, so this library defines one:
 *   code   = OCP E4M3 ("fn": bias 7, subnormals, max 448, S.1111.111 NaN) of
 *            c / s_t, rounded to nearest even, saturated to +-448;
 *   s_t    = 2^e_t per token, e_t the smallest integer with
 *            max_i |c_t[i]| <= 448 * 2^e_t, clamped to [-15, 7] (division by
 *            s_t is exact; code * s_t is exactly an IEEE half);
 *   k_pe   = IEEE half (f16), rounded to nearest even.
 * Block layout (block_size tokens, all little-endian):
 *   block_size rows of (kv_lora_rank + 2 * rope_dim) bytes: the codes, then
 *   the f16 k_pe; then block_size fp32 scales s_t.
 * DeepSeek-V3: 41216 bytes per 64-token block (644 per token; bf16: 1152).
 * Dequantised cache: c~ = value(code) * s_t, k_pe~ = the f16 value; the
 * decode over an FP8 pool computes the absorbed attention of that cache.
 * kv_lora_rank must be a multiple of 16, rope_dim of 8, block_size of 4. */

/* Bytes of one FP8 cache block; 0 for unsupported dims. */
MLA_API size_t mla_fp8_block_bytes(const mla_dims_t* dims);

/* Converts a bf16 pool (num_blocks blocks, layout above) into the FP8 layout:
 * every row, the unused ones included (rows must hold finite values; a NaN
 * gives NaN codes). pool bf16 [num_blocks, block_size, d_c + d_r] and
 * pool_fp8 (num_blocks * mla_fp8_block_bytes bytes), both 16-byte aligned,
 * not overlapping. */
MLA_API int mla_cache_to_fp8(const mla_dims_t* dims, const void* pool, int64_t num_blocks, void* pool_fp8,
                             void* stream);

/* ------------------------------------------------------------------ */
/* Cache append: [MLA-arch] 2.2 (kv_a_proj_with_mqa, kv_a_layernorm) and
 * 4.2 (RoPE fused with the cache update); RoPE as in [MQA-MLA] "MLA的实现".
 *   kv   = x . w_kva                       (fp32 accumulate)
 *   c    = kv[:d_c] / sqrt(mean(kv[:d_c]^2) + rms_eps) * gamma
 *   k_pe = rotate-half RoPE of kv[d_c:] at positions[i], base rope_base
 *   pool[row(seq_ids[i], positions[i])] = bf16(c) ++ bf16(k_pe)
 * Arguments:
 *   x          bf16 [n_tokens, hidden]
 *   w_kva      bf16 [hidden, kv_lora_rank + rope_dim]
 *   rms_gamma  bf16 [kv_lora_rank] or NULL (= ones)
 *   seq_ids    int32 [n_tokens] in [0, num_seqs), positions int32 [n_tokens]
 *   block_table int32 [num_seqs, max_blocks_per_seq]; pool as above (written
 *              only at the target rows)
 *   workspace  >= mla_append_workspace_size(dims, n_tokens, hidden) bytes,
 *              256-byte aligned, contents need not be initialised.
 * A (seq, position) whose sequence is outside [0, num_seqs), whose page is
 * missing (-1 / >= num_blocks) or outside max_blocks_per_seq is skipped and
 * flags MLA_ERR_DEVICE_FAULT. Rows of distinct tokens must not coincide. */
MLA_API int mla_append_kv(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden,
                  const void* w_kva, const void* rms_gamma, float rms_eps, float rope_base,
                  const int32_t* seq_ids, const int32_t* positions,
                  const int32_t* block_table, int32_t num_seqs, int32_t max_blocks_per_seq,
                  void* pool, int64_t num_blocks,
                  void* workspace, size_t workspace_bytes, void* stream);

MLA_API size_t mla_append_workspace_size(const mla_dims_t* dims, int32_t n_tokens, int32_t hidden);

/* mla_append_kv into the FP8 cache: the same arguments and checks, pool_fp8
 * in the FP8 layout. c is rounded to bf16 (the value the bf16 cache would
 * store) and then quantised with its token's scale; k_pe is rounded to f16
 * from fp32. The workspace size is mla_append_workspace_size's. */
MLA_API int mla_append_kv_fp8(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden,
                              const void* w_kva, const void* rms_gamma, float rms_eps, float rope_base,
                              const int32_t* seq_ids, const int32_t* positions,
                              const int32_t* block_table, int32_t num_seqs, int32_t max_blocks_per_seq,
                              void* pool_fp8, int64_t num_blocks,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Query projection of new tokens, the step before the absorption:
 * [MLA-arch] 2.1 (q_a_proj hidden -> q_lora_rank, q_a_layernorm, q_b_proj
 * q_lora_rank -> H * qk_head_dim) and 1 (qk_head_dim = the d_n non-RoPE part
 * followed by the d_r RoPE part); RoPE as in [MQA-MLA] "MLA的实现".
 *   c_q   = x . w_qa / sqrt(mean((x . w_qa)^2) + rms_eps) * q_gamma
 *   q     = bf16(c_q) . w_qb, viewed as [n_tokens, H, d_n + d_r]
 *   q_nope[t, h, :] = bf16(q[t, h, :d_n])
 *   q_pe[t, h, :]   = bf16(rotate-half RoPE of q[t, h, d_n:] at positions[t])
 * Arguments:
 *   x        bf16 [n_tokens, hidden], 16-byte aligned
 *   w_qa     bf16 [hidden, q_rank], 16-byte aligned
 *   q_gamma  bf16 [q_rank] or NULL (= ones)
 *   w_qb     bf16 [q_rank, H * (qk_nope_dim + rope_dim)], 16-byte aligned
 *   positions int32 [n_tokens] on the device (absolute token positions)
 *   q_nope   bf16 [n_tokens, H, qk_nope_dim] (output; the layout mla_decode
 *            takes with n_tokens = batch * q_len)
 *   q_pe     bf16 [n_tokens, H, rope_dim] (output)
 *   workspace >= mla_q_proj_workspace_size(dims, n_tokens, hidden, q_rank)
 *            bytes, 256-byte aligned, contents need not be initialised.
 * hidden, q_rank and H * (qk_nope_dim + rope_dim) must be multiples of 64,
 * q_rank <= 2048 and rope_dim even and <= 128 (else MLA_ERR_UNSUPPORTED_DIMS). Accumulation is
 * fp32; c_q is rounded to bf16 before the second product. With rope_dim 64
 * and qk_nope_dim a multiple of 64 (DeepSeek-V3) the second product writes
 * the heads itself and q_nope and q_pe must be 16-byte aligned
 * (MLA_ERR_INVALID_ARG otherwise). */
MLA_API int mla_q_proj(const mla_dims_t* dims, const void* x, int32_t n_tokens, int32_t hidden,
                       const void* w_qa, int32_t q_rank, const void* q_gamma, float rms_eps,
                       const void* w_qb, const int32_t* positions, float rope_base,
                       void* q_nope, void* q_pe, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace mla_q_proj needs; 0 if the arguments are invalid or the
 * dims unsupported. */
MLA_API size_t mla_q_proj_workspace_size(const mla_dims_t* dims, int32_t n_tokens, int32_t hidden,
                                         int32_t q_rank);

/* ------------------------------------------------------------------ */
/* Absorbed decode: [MQA-MLA] "MLA的实现" forward_inference_absorbed with the
 * query absorption of [MLA-arch] 3.1, restated for q_len new tokens per
 * sequence over the paged cache. For sequence b (context_lens[b] = L
 * cached tokens, the q_len new ones included), new token s, head h:
 *   q_lat  = W_UK[h]^T q_nope[b,s,h]                       (d_c)
 *   z_t    = scale * (q_lat . c_t + q_pe[b,s,h] . k_pe_t),  t = 0 .. L-q_len+s
 *   o_lat  = softmax(z) . c                                 (d_c)
 *   out[b,s,h] = W_UV[h] o_lat                              (d_v)
 * computed as split-KV partials merged by a log-sum-exp combine.
 * Arguments:
 *   q_nope  bf16 [batch, q_len, H, qk_nope_dim]
 *   q_pe    bf16 [batch, q_len, H, rope_dim]   (RoPE already applied)
 *   pool, block_table: as above (read only)
 *   context_lens int32 [batch] on the device; every value must be in
 *           [q_len, max_context_len] and covered by the block table
 *   max_context_len  host int, an upper bound of context_lens (sizes the
 *           launch and the workspace)
 *   w_uk    bf16 [H, qk_nope_dim, kv_lora_rank]
 *   w_uv    bf16 [H, v_head_dim, kv_lora_rank]
 *   out     bf16 [batch, q_len, H, v_head_dim]
 *   workspace >= mla_decode_workspace_size(...) bytes, 256-byte aligned,
 *           contents need not be initialised
 *   opts    NULL or kernel / split overrides
 * Alignment: q_nope, q_pe, w_uk, w_uv and out 16-byte aligned (with d_n a
 * multiple of 64, d_c of 256, d_r of 8, d_v of 16) select the tcgen05
 * absorption, merge and up-projection kernels; otherwise CUDA-core kernels
 * run them. The tcgen05 attention kernel (opts->kernel = 1, the default for
 * DeepSeek-V3 dims) needs the tcgen05 kernels around it and returns
 * MLA_ERR_INVALID_ARG when they do not apply.
 * Rounding: q_lat is rounded to bf16 before the score product and the
 * softmax weights to bf16 before the value product; accumulation and the
 * combine are fp32; split partials are fp32 (CUDA-core kernel) or rounded
 * to bf16 (tcgen05 kernel); o_lat is rounded to bf16 before the
 * up-projection and out to bf16 once. With the FP8 cache (opts->cache_fp8)
 * q_lat, q_pe and the softmax weights are rounded to f16 instead, and the
 * cache enters the products as its exact dequantised f16 values. */
MLA_API int mla_decode(const mla_dims_t* dims, const void* q_nope, const void* q_pe,
               int32_t batch, int32_t q_len,
               const void* pool, int64_t num_blocks,
               const int32_t* block_table, int32_t max_blocks_per_seq,
               const int32_t* context_lens, int32_t max_context_len,
               const void* w_uk, const void* w_uv, void* out,
               void* workspace, size_t workspace_bytes,
               const mla_decode_opts_t* opts, void* stream);

MLA_API size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t batch, int32_t q_len,
                                 int32_t max_context_len, const mla_decode_opts_t* opts);

/* ------------------------------------------------------------------ */
/* mla_decode for callers that cannot allocate device memory. The paper
 * has no counterpart: this is a deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc (or any allocator): a plugin whose
 * host process owns all device memory through its own pooled allocator and
 * forbids raw allocations, a latency-critical path that cannot afford the
 * device-wide synchronisation cudaMalloc/cudaFree may cause, or plain C code
 * with no memory manager at all. They still pass every input and output
 * buffer; only the decode scratch (split-KV schedule, absorbed queries and
 * partial results, the same bytes mla_decode_workspace_size() reports) comes
 * from a fixed buffer compiled into the library: a static device array of
 * MLA_NO_ALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits.
 *
 * Arguments and results are those of mla_decode without the workspace.
 * Returns MLA_ERR_SCRATCH_LIMIT, before enqueuing anything, when the
 * problem needs more scratch than the buffer holds (for DeepSeek-V3 dims
 * the default schedule fits batch * q_len up to 64).
 *
 * Set-up: the first call in each CUDA context (the device's primary
 * context for runtime users) looks up the buffer's device address
 * (cudaGetSymbolAddress, with that context current) and caches it under the
 * context's unique id, so a new context -- another device, a driver-API
 * context, the primary context re-created after cudaDeviceReset -- gets its
 * own look-up. Make that first call before any stream capture.
 * Sharing: every call on a device uses the same buffer and leaves its
 * contents behind. Nothing in it needs to start at zero (each call writes
 * every scratch byte it later reads), but calls whose work overlaps on the
 * GPU (different streams, no ordering between them) race on the buffer:
 * order them on one stream or with events. */
#define MLA_NO_ALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)

MLA_API int mla_decode_no_alloc(const mla_dims_t* dims, const void* q_nope, const void* q_pe,
                                int32_t batch, int32_t q_len,
                                const void* pool, int64_t num_blocks,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* context_lens, int32_t max_context_len,
                                const void* w_uk, const void* w_uv, void* out,
                                const mla_decode_opts_t* opts, void* stream);

/* ------------------------------------------------------------------ */
/* Output projection: y = x W for a few token rows, the step after the
 * attention ([MQA-MLA] "MLA的实现": the W_O of forward_training and the
 * W_o_absorbed of forward_inference_absorbed; [MLA-arch] 3.1, W_V absorbed
 * into the O projection). Two uses:
 *   x = out viewed as [n_tokens, H * v_head_dim], w = W_O [H * v_head_dim,
 *       hidden] (row h * v_head_dim + d holds head h's value index d): the
 *       output projection after the per-head up-projection;
 *   x = o_lat viewed as [n_tokens, H * kv_lora_rank] (mla_decode with
 *       output_latent = 1), w = W_UV^T W_O stacked per head [H * kv_lora_rank,
 *       hidden]: the full absorption, which reads kv_lora_rank / v_head_dim
 *       times the weight bytes.
 *   y[t, n] = bf16(sum_k x[t, k] w[k, n]), fp32 accumulation.
 * Arguments:
 *   x  bf16 [n_tokens, k], 16-byte aligned;  w  bf16 [k, n], 16-byte aligned
 *   y  bf16 [n_tokens, n], 8-byte aligned
 *   workspace >= mla_o_proj_workspace_size(n_tokens, k, n) bytes, 256-byte
 *            aligned, contents need not be initialised.
 * k and n must be multiples of 64 (else MLA_ERR_UNSUPPORTED_DIMS). */
MLA_API int mla_o_proj(const void* x, int32_t n_tokens, int32_t k, const void* w, int32_t n, void* y,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace mla_o_proj needs; 0 if the sizes are invalid. */
MLA_API size_t mla_o_proj_workspace_size(int32_t n_tokens, int32_t k, int32_t n);

/* ------------------------------------------------------------------ */
/* Log-sum-exp combine of split-KV partials (the merge the split decode
 * needs; no page states it, it is exact softmax algebra). For group g
 * (= b*q_len + s) and head h, with parts i in [part_offsets[g],
 * part_offsets[g+1]):
 *   M = max_i lse_i;  w_i = exp(lse_i - M)  (0 when lse_i = -inf)
 *   o_lat[g,h] = sum_i w_i o_part[i,h] / sum_i w_i
 *   lse_out[g,h] = M + log(sum_i w_i)
 * A group whose parts all have lse = -inf (or that has none) gets zeros and
 * lse = -inf.
 *   o_part   fp32 [n_parts, H, kv_lora_rank]   (each part normalised)
 *   lse_part fp32 [n_parts, H]                 (natural log)
 *   part_offsets int32 [n_groups + 1], non-decreasing, device memory
 *   o_lat    fp32 [n_groups, H, kv_lora_rank]
 *   lse_out  fp32 [n_groups, H] or NULL */
MLA_API int mla_combine(const mla_dims_t* dims, const float* o_part, const float* lse_part,
                const int32_t* part_offsets, int32_t n_groups,
                float* o_lat, float* lse_out, void* stream);

/* ------------------------------------------------------------------ */
/* Test hook: the pool row of (seq_ids[i], positions[i]) from the same
 * device resolver the append and decode kernels use; -1 where the sequence,
 * page or block id is out of range. rows: int64 [n] device. */
MLA_API int mla_debug_resolve_slots(const mla_dims_t* dims, const int32_t* block_table, int32_t num_seqs,
                            int32_t max_blocks_per_seq, int64_t num_blocks,
                            const int32_t* seq_ids, const int32_t* positions, int32_t n,
                            int64_t* rows, void* stream);

/* Reads and clears the device error word of the current device after
 * synchronising `stream`. *device_status receives MLA_OK or the first
 * MLA_ERR_DEVICE_* recorded since the last call. */
MLA_API int mla_get_device_error(int* device_status, void* stream);

/* Static description of a status code (never NULL). */
MLA_API const char* mla_error_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
MLA_API int mla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
