"""fp64 CPU oracle for MLA decode over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY. This module is the independent checker of the CUDA
library. Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it; the library never does, and it shares no
code with the library (inputs come from ``mla_latent_kv_29_b200.inputs``,
which draws random numbers only).

Sources (cited by page title and section):

* [MLA-arch] "MLA架构：低秩注意力机制优化LLM显存与计算效率"
  (intelliparadigm.com) -- section 1 (128 heads, qk_head_dim = 128 nope +
  64 rope, RoPE part shared by all heads), section 2.1 (q_a_proj hidden ->
  q_lora_rank, q_a_layernorm, q_b_proj -> H * qk_head_dim), section 2.2 (kv_a_proj_with_mqa
  hidden -> kv_lora_rank + rope, kv_a_layernorm = RMSNorm(kv_lora_rank),
  kv_b_proj -> per-head K-nope and V), section 3.1 (absorption is matrix
  associativity), section 3.2 (cache = c_kv [bsz, seq, 512] + pe
  [bsz, seq, 64]), section 4.2 (fuse RoPE with the cache update).
* [MQA-MLA] "一次讲透MHA、GQA、MQA、MLA" (xxmr.cn) -- section "MLA的实现":
  the RoPE module (rotate-half, inv_freq = 1/theta^(2i/d), cos/sin built
  from the frequencies repeated twice), ``forward_training`` (explicit
  decompression: K = [W_UK c ; RoPE(k_r)], V = W_UV c, scale =
  (d_head + d_rope)^-1/2, softmax, P V) and ``forward_inference_absorbed``
  (scores = q_absorbed . c_kv + q_r . k_r, output = P . c_kv then the
  up-projection); section "测试与结果验证" (the two forms agree).
* [R1V3-MLA] the DeepSeek R1/V3 MLA article (mlqm.cn/news/500296),
  section 2.3 (weight absorption removes the explicit K/V expansion).

Everything is computed in float64 from the exact values the GPU receives
(bf16 storage upcast exactly). Readings where the pages are silent or
garbled:

* causal rule for several new tokens: query s of a sequence with L cached
  tokens (the Sq new ones included) sees tokens 0 .. L - Sq + s;
* RMSNorm eps = 1e-6 and gamma = ones unless given;
* RoPE positions are absolute token indices; base 10000; rotate-half pairs
  (i, i + d/2);
* the cache row is c_kv followed by k_pe (the split order of the joint
  projection output);
* W_UK[h] and W_UV[h] are [d_head, d_c] so that k_nope = W_UK[h] c and
  v = W_UV[h] c (the ``view(H, D_h, D_c)`` of the absorbed listing);
* combine of split-KV partials: o = sum_i e^{lse_i - M} o_i /
  sum_i e^{lse_i - M}, lse = M + log sum_i e^{lse_i - M}; a partition with
  no token carries lse = -inf and weight 0.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -math.inf


def _f64(a) -> np.ndarray:
    """Exact upcast of a torch tensor (any float dtype) or array to float64."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- RoPE ----
def rope_inv_freq(rope_dim: int, base: float = 10000.0) -> np.ndarray:
    """[MQA-MLA] "MLA的实现", RoPE module: inv_freq_i = base^(-2i/d), i < d/2."""
    i = np.arange(0, rope_dim, 2, dtype=np.float64)
    return 1.0 / (base ** (i / rope_dim))


def rope(x, positions, base: float = 10000.0) -> np.ndarray:
    """Rotate-half RoPE of [MQA-MLA] "MLA的实现".

    x [..., d] at integer positions [...] (broadcast against x's leading
    dims). cos/sin use the frequency vector repeated twice; the result is
    x*cos + rotate_half(x)*sin with rotate_half(x) = (-x2, x1).
    """
    x = _f64(x)
    d = x.shape[-1]
    pos = np.asarray(positions, dtype=np.float64)
    freqs = pos[..., None] * rope_inv_freq(d, base)  # [..., d/2]
    emb = np.concatenate([freqs, freqs], axis=-1)  # [..., d]
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    rot = np.concatenate([-x2, x1], axis=-1)
    return x * np.cos(emb) + rot * np.sin(emb)


# ------------------------------------------------------------- RMSNorm ----
def rmsnorm(v, gamma=None, eps: float = 1e-6) -> np.ndarray:
    """kv_a_layernorm of [MLA-arch] 2.2: v / sqrt(mean(v^2) + eps) * gamma."""
    v = _f64(v)
    r = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    out = v * r
    if gamma is not None:
        out = out * _f64(gamma)
    return out


# --------------------------------------------------------- paging -------
def resolve_slot(block_table, b: int, t: int, block_size: int) -> int:
    """Pool row of token t of sequence b: table[b][t // bs] * bs + t % bs."""
    return int(block_table[b][t // block_size]) * block_size + t % block_size


def gather_sequence(pool, block_table, b: int, length: int, dims):
    """Rows 0..length-1 of sequence b from the paged pool.

    pool is [num_blocks, block_size, d_c + d_r] (any float dtype); returns
    (c [L, d_c], k_pe [L, d_r]) float64, the cache of [MLA-arch] 3.2.
    """
    bs = dims.block_size
    flat = pool.reshape(-1, pool.shape[-1])
    rows = [resolve_slot(block_table, b, t, bs) for t in range(length)]
    r = _f64(flat[rows]) if len(rows) else np.zeros((0, flat.shape[-1]))
    return r[:, : dims.kv_lora_rank], r[:, dims.kv_lora_rank:]


# ------------------------------------------------------------ append ----
def append_rows(x, w_kva, positions, kv_lora_rank: int, gamma=None,
                eps: float = 1e-6, base: float = 10000.0) -> np.ndarray:
    """New cache rows from hidden states: [MLA-arch] 2.2 and 4.2.

    kv = x . W_kva (the bias-free joint down-projection, [hidden, d_c + d_r]),
    c = RMSNorm(kv[:, :d_c]), k_pe = RoPE(kv[:, d_c:], position); the stored
    row is c followed by k_pe. Returns float64 [T, d_c + d_r].
    """
    kv = _f64(x) @ _f64(w_kva)
    c = rmsnorm(kv[:, :kv_lora_rank], gamma, eps)
    k_pe = rope(kv[:, kv_lora_rank:], np.asarray(positions), base)
    return np.concatenate([c, k_pe], axis=-1)


# ---------------------------------------------------- query projection ----
def query_projection(x, w_qa, w_qb, positions, num_heads: int, qk_nope_dim: int, rope_dim: int,
                     gamma=None, eps: float = 1e-6, base: float = 10000.0):
    """Queries of new tokens from their hidden states: [MLA-arch] 2.1 and 1.

    c_q = RMSNorm(x . W_qa) (q_a_proj, hidden -> q_lora_rank, then
    q_a_layernorm), q = c_q . W_qb (q_b_proj, q_lora_rank -> H * qk_head_dim),
    each head's qk_head_dim values being the d_n non-RoPE part followed by the
    d_r RoPE part (section 1 names them in that order); the RoPE part is
    rotated at the token's position. Returns float64 (q_nope [T, H, d_n],
    q_pe [T, H, d_r]).
    """
    c_q = rmsnorm(_f64(x) @ _f64(w_qa), gamma, eps)
    q = (c_q @ _f64(w_qb)).reshape(c_q.shape[0], num_heads, qk_nope_dim + rope_dim)
    pos = np.asarray(positions)
    return q[..., :qk_nope_dim], rope(q[..., qk_nope_dim:], pos[:, None], base)


# ------------------------------------------------------------ decode ----
def visible_count(length: int, q_len: int, s: int) -> int:
    """Tokens visible to new-token s: 0 .. length - q_len + s (inclusive)."""
    return length - q_len + s + 1


def decode_sequence(q_nope, q_pe, c, k_pe, w_uk, w_uv, scale: float,
                    return_probs: bool = False):
    """Explicit (decompressed) MLA attention for one sequence.

    Follows ``forward_training`` of [MQA-MLA] "MLA的实现" restated for the
    Sq newest tokens: per head h, K_h = [c W_UK[h]^T ; k_pe] (k_pe shared
    by all heads, [MLA-arch] 1), V_h = c W_UV[h]^T, z = scale * Q_h K_h^T
    with the causal rule above, p = softmax(z), out = p V_h.

    q_nope [Sq, H, d_n], q_pe [Sq, H, d_r], c [L, d_c], k_pe [L, d_r],
    w_uk [H, d_n, d_c], w_uv [H, d_v, d_c]. Returns out [Sq, H, d_v]
    (and p [Sq, H, L] with exact zeros on masked tokens if asked).
    """
    q_nope, q_pe, c, k_pe = _f64(q_nope), _f64(q_pe), _f64(c), _f64(k_pe)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    sq, H = q_nope.shape[0], q_nope.shape[1]
    L = c.shape[0]
    dv = w_uv.shape[1]
    out = np.zeros((sq, H, dv))
    probs = np.zeros((sq, H, L)) if return_probs else None
    for h in range(H):
        k_h = np.concatenate([c @ w_uk[h].T, k_pe], axis=1)  # [L, d_n + d_r]
        v_h = c @ w_uv[h].T  # [L, d_v]
        for s in range(sq):
            n = visible_count(L, sq, s)
            q = np.concatenate([q_nope[s, h], q_pe[s, h]])
            z = scale * (k_h[:n] @ q)
            p = np.exp(z - z.max())
            p /= p.sum()
            out[s, h] = p @ v_h[:n]
            if return_probs:
                probs[s, h, :n] = p
    return (out, probs) if return_probs else out


def decode_paged(q_nope, q_pe, pool, block_table, lengths, w_uk, w_uv, dims,
                 scale: float, batch_ids=None):
    """Decode output [B, Sq, H, d_v] float64 over the paged pool.

    ``batch_ids`` restricts the work to some sequences (the rows of the other
    sequences are left as NaN) so that large workloads can be checked on a
    sample.
    """
    q_nope, q_pe = _f64(q_nope), _f64(q_pe)
    B, sq, H = q_nope.shape[:3]
    out = np.full((B, sq, H, _f64(w_uv).shape[1]), np.nan)
    ids = range(B) if batch_ids is None else batch_ids
    lengths = [int(v) for v in (lengths.tolist() if hasattr(lengths, "tolist") else lengths)]
    for b in ids:
        c, kpe = gather_sequence(pool, block_table, b, lengths[b], dims)
        out[b] = decode_sequence(q_nope[b], q_pe[b], c, kpe, w_uk, w_uv, scale)
    return out


# ----------------------------------------------- split-KV and combine ----
def latent_partial(q_lat, q_pe, c, k_pe, scale: float):
    """Absorbed-form attention of one head over a token subset.

    The latent-space state the split-KV path carries: scores
    z_t = scale (q_lat . c_t + q_pe . k_pe_t) as in
    ``forward_inference_absorbed`` of [MQA-MLA], o = softmax(z) . c over
    the subset, lse = log sum_t e^{z_t}. An empty subset gives
    (zeros, -inf).
    """
    q_lat, q_pe, c, k_pe = _f64(q_lat), _f64(q_pe), _f64(c), _f64(k_pe)
    if c.shape[0] == 0:
        return np.zeros(c.shape[1]), NEG_INF
    z = scale * (c @ q_lat + k_pe @ q_pe)
    m = z.max()
    e = np.exp(z - m)
    s = e.sum()
    return (e @ c) / s, m + math.log(s)


def merge_partials(o_parts, lse_parts):
    """Log-sum-exp merge of split-KV partials (the combine step).

    o_parts [n, ..., d], lse_parts [n, ...]. Returns (o [..., d], lse [...]).
    Partitions with lse = -inf get weight 0; if every partition is empty the
    result is zeros with lse = -inf.
    """
    o = _f64(o_parts)
    lse = _f64(lse_parts)
    m = np.max(lse, axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w = np.where(np.isfinite(lse), np.exp(lse - safe_m[None]), 0.0)
    den = w.sum(axis=0)
    num = np.einsum("n...,n...d->...d", w, o)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
        lse_out = np.where(den > 0, safe_m + np.log(np.where(den > 0, den, 1.0)), NEG_INF)
    return out, lse_out


def absorb_query(q_nope, w_uk) -> np.ndarray:
    """q_lat[..., h, :] = W_UK[h]^T q_nope[..., h, :] (absorption into the query)."""
    return np.einsum("...hn,hnc->...hc", _f64(q_nope), _f64(w_uk))


def up_project(o_lat, w_uv) -> np.ndarray:
    """out[..., h, :] = W_UV[h] o_lat[..., h, :] (the value up-projection)."""
    return np.einsum("...hc,hvc->...hv", _f64(o_lat), _f64(w_uv))


# --------------------------------------------------- output projection ----
def output_projection(out, w_o) -> np.ndarray:
    """y = concat_h(out[..., h, :]) . W_O, the projection after the per-head
    up-projection ([MQA-MLA] "MLA的实现": forward_training ends with w_o over
    the heads' outputs laid side by side; [MLA-arch] 3.1).

    out [..., H, d_v]; w_o [H * d_v, hidden], row h * d_v + d holding head h's
    value index d (the page's linear weight viewed as [D_model, N_h, D_h],
    transposed). Returns float64 [..., hidden].
    """
    o = _f64(out)
    return o.reshape(o.shape[:-2] + (-1,)) @ _f64(w_o)


def absorbed_output_weight(w_uv, w_o) -> np.ndarray:
    """W_UV absorbed into the output projection, stacked per head.

    Block h (rows h * d_c .. (h + 1) * d_c - 1) is W_UV[h]^T . W_O[h * d_v ..
    (h + 1) * d_v - 1] ([MQA-MLA] forward_inference_absorbed, the einsum that
    fuses w_uv into w_o; [MLA-arch] 3.1, W_V absorbed into the O projection),
    so that o_lat[..., H, d_c] flattened times this weight is the output
    projection of the up-projected heads. Returns float64 [H * d_c, hidden].
    """
    wv, wo = _f64(w_uv), _f64(w_o)
    H, dv, _ = wv.shape
    return np.concatenate([wv[h].T @ wo[h * dv:(h + 1) * dv] for h in range(H)], axis=0)


def decode_latent_paged(q_nope, q_pe, pool, block_table, lengths, w_uk, dims, scale: float,
                        batch_ids=None) -> np.ndarray:
    """o_lat [B, Sq, H, d_c] float64: the attention output in the latent space
    (softmax of the absorbed scores applied to c, [MQA-MLA]
    forward_inference_absorbed before its output einsum), per new token with
    the causal rule above. Rows of sequences outside ``batch_ids`` are NaN."""
    q_lat = absorb_query(q_nope, w_uk)
    qp = _f64(q_pe)
    B, sq, H = q_lat.shape[:3]
    out = np.full((B, sq, H, dims.kv_lora_rank), np.nan)
    ids = range(B) if batch_ids is None else batch_ids
    lengths = [int(v) for v in (lengths.tolist() if hasattr(lengths, "tolist") else lengths)]
    for b in ids:
        c, kpe = gather_sequence(pool, block_table, b, lengths[b], dims)
        for s in range(sq):
            n = visible_count(lengths[b], sq, s)
            for h in range(H):
                out[b, s, h], _ = latent_partial(q_lat[b, s, h], qp[b, s, h], c[:n], kpe[:n], scale)
    return out
