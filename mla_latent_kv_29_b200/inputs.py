"""Seeded synthetic inputs for MLA decode workloads.

This module only draws random numbers and lays them out: context lengths,
shuffled block tables, N(0, sigma^2) tensors and their bf16 storage copies.
It holds none of the attention arithmetic (no RMSNorm, no RoPE, no softmax,
no projection), so the fp64 oracle and the CUDA path can both consume what
it produces without sharing any computation.

Workload shapes follow the DeepSeek-V3 MLA dimensions described on the page
"MLA架构：低秩注意力机制优化LLM显存与计算效率" (section 1: 128 heads,
qk_head_dim 128 + 64; section 2.2: kv_a_proj_with_mqa 7168 -> 512 + 64) and
the per-token latent cache of section 3.2 (c_kv 512 + shared pe 64).

Every random stream is a torch CPU ``Generator`` seeded from the workload
seed plus a fixed per-tensor salt, so a tensor can be regenerated on its own
(for example one sequence's cache rows) without drawing the others.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK_SIZE = 64  # tokens per cache page


@dataclasses.dataclass(frozen=True)
class Dims:
    """Per-layer MLA sizes (names follow the DeepSeek-V3 config keys)."""

    num_heads: int
    kv_lora_rank: int  # d_c, latent width stored per token
    rope_dim: int  # d_r, decoupled RoPE key width stored per token
    qk_nope_dim: int  # d_n, per-head non-RoPE query/key width
    v_head_dim: int  # d_v, per-head value width
    block_size: int = BLOCK_SIZE

    @property
    def row_width(self) -> int:
        """Values stored per cached token: c_kv followed by k_pe."""
        return self.kv_lora_rank + self.rope_dim


V3 = Dims(num_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope_dim=128, v_head_dim=128)
TINY = Dims(num_heads=16, kv_lora_rank=64, rope_dim=16, qk_nope_dim=32, v_head_dim=32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    ``kv_values`` is "normal" when cache rows are raw N(0,1) draws, and
    "rmsnorm_rope" when the raw draws are meant to be passed through the
    cache-append normalisation (RMSNorm on c_kv, RoPE on k_pe at the token's
    position) before being stored; the generator itself never applies them.
    """

    name: str
    dims: Dims
    batch: int
    q_len: int
    length_range: tuple  # (lo, hi) inclusive; lo == hi for fixed lengths
    softmax_scale: float
    w_std: float  # std of W_UK / W_UV entries
    paged: bool  # False: one block per sequence, identity table
    kv_values: str
    seed: int
    append_hidden: int = 0  # >0: the last q_len tokens of each sequence come from an append
    append_w_std: float = 0.0
    spare_blocks: int = 0  # unused pool blocks (filled with sentinels by tests)


def _tiny() -> Workload:
    return Workload(
        name="tiny_b1_l128",
        dims=dataclasses.replace(TINY, block_size=128),
        batch=1,
        q_len=1,
        length_range=(128, 128),
        softmax_scale=1.0 / math.sqrt(48.0),
        w_std=math.sqrt(1.0 / 64.0),
        paged=False,
        kv_values="normal",
        seed=1000,
    )


WORKLOADS = {
    "tiny_b1_l128": _tiny(),
    "v3_b1_l4096": Workload(
        name="v3_b1_l4096", dims=V3, batch=1, q_len=1, length_range=(4096, 4096),
        softmax_scale=1.0 / math.sqrt(192.0), w_std=math.sqrt(1.0 / 512.0), paged=True,
        kv_values="rmsnorm_rope", seed=1001),
    "v3_b64_l1k_8k": Workload(
        name="v3_b64_l1k_8k", dims=V3, batch=64, q_len=1, length_range=(1024, 8192),
        softmax_scale=1.0 / math.sqrt(192.0), w_std=math.sqrt(1.0 / 512.0), paged=True,
        kv_values="rmsnorm_rope", seed=1002),
    "v3_b8_l32k": Workload(
        name="v3_b8_l32k", dims=V3, batch=8, q_len=1, length_range=(32768, 32768),
        softmax_scale=1.0 / math.sqrt(192.0), w_std=math.sqrt(1.0 / 512.0), paged=True,
        kv_values="rmsnorm_rope", seed=1003),
    "v3_b16_sq4_l16k_append": Workload(
        name="v3_b16_sq4_l16k_append", dims=V3, batch=16, q_len=4,
        length_range=(16384, 16384), softmax_scale=1.0 / math.sqrt(192.0),
        w_std=math.sqrt(1.0 / 512.0), paged=True, kv_values="rmsnorm_rope", seed=1004,
        append_hidden=7168, append_w_std=math.sqrt(1.0 / 7168.0)),
    # fixed-length variant of the batched workload (batch 64, 8K context each)
    "v3_b64_l8k": Workload(
        name="v3_b64_l8k", dims=V3, batch=64, q_len=1, length_range=(8192, 8192),
        softmax_scale=1.0 / math.sqrt(192.0), w_std=math.sqrt(1.0 / 512.0), paged=True,
        kv_values="rmsnorm_rope", seed=1005),
    # chunked prefill: 4 sequences each append a chunk of 128 prompt tokens
    # (positions 3968..4095) and attend causally over their 4096-token context
    "v3_b4_sq128_l4k_prefill": Workload(
        name="v3_b4_sq128_l4k_prefill", dims=V3, batch=4, q_len=128,
        length_range=(4096, 4096), softmax_scale=1.0 / math.sqrt(192.0),
        w_std=math.sqrt(1.0 / 512.0), paged=True, kv_values="rmsnorm_rope", seed=1006,
        append_hidden=7168, append_w_std=math.sqrt(1.0 / 7168.0)),
}

# Salts for independent streams.
_S_LEN, _S_TABLE, _S_Q_NOPE, _S_Q_PE, _S_W_UK, _S_W_UV = 1, 2, 3, 4, 5, 6
_S_X, _S_W_KVA, _S_GAMMA = 7, 8, 9
_S_QX, _S_W_QA, _S_W_QB, _S_QGAMMA, _S_QPOS = 10, 11, 12, 13, 14
_S_CACHE = 1 << 20  # + sequence index


def generator(seed: int, salt: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((int(seed) * 1_000_003 + int(salt)) % (1 << 62))
    return g


def normal(shape, std: float, seed: int, salt: int) -> torch.Tensor:
    """fp32 N(0, std^2) draws from the (seed, salt) stream."""
    t = torch.randn(*shape, generator=generator(seed, salt), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def bf16(t: torch.Tensor) -> torch.Tensor:
    """Storage copy: round to bfloat16 (round-to-nearest-even)."""
    return t.to(torch.bfloat16)


def context_lengths(w: Workload) -> torch.Tensor:
    """[B] int32 context lengths, each including the q_len newest tokens."""
    lo, hi = w.length_range
    if lo == hi:
        return torch.full((w.batch,), lo, dtype=torch.int32)
    return torch.randint(lo, hi + 1, (w.batch,), generator=generator(w.seed, _S_LEN),
                         dtype=torch.int64).to(torch.int32)


def block_table(w: Workload, lengths: torch.Tensor):
    """Block table [B, max_blocks] int32 and pool size in blocks.

    Paged workloads draw one global permutation of the pool's block ids and
    hand them out to sequences in order (so consecutive pages of a sequence
    land at random pool positions). Unused table entries are -1. Contiguous
    workloads give sequence b the single block b.
    """
    bs = w.dims.block_size
    nblk = [(int(L) + bs - 1) // bs for L in lengths.tolist()]
    max_blocks = max(nblk) if nblk else 0
    total = sum(nblk) + w.spare_blocks
    table = torch.full((w.batch, max(max_blocks, 1)), -1, dtype=torch.int32)
    if w.paged:
        perm = torch.randperm(total, generator=generator(w.seed, _S_TABLE)).to(torch.int32)
    else:
        perm = torch.arange(total, dtype=torch.int32)
    k = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[k:k + n]
        k += n
    return table, total


def queries(w: Workload):
    """q_nope [B, Sq, H, d_n] and q_pe [B, Sq, H, d_r], fp32 N(0,1).

    q_pe is taken as already rotated: RoPE is orthogonal, so a rotated
    N(0, I) vector is again N(0, I).
    """
    d = w.dims
    q_nope = normal((w.batch, w.q_len, d.num_heads, d.qk_nope_dim), 1.0, w.seed, _S_Q_NOPE)
    q_pe = normal((w.batch, w.q_len, d.num_heads, d.rope_dim), 1.0, w.seed, _S_Q_PE)
    return q_nope, q_pe


def up_weights(w: Workload):
    """W_UK [H, d_n, d_c] and W_UV [H, d_v, d_c], fp32 N(0, w_std^2)."""
    d = w.dims
    w_uk = normal((d.num_heads, d.qk_nope_dim, d.kv_lora_rank), w.w_std, w.seed, _S_W_UK)
    w_uv = normal((d.num_heads, d.v_head_dim, d.kv_lora_rank), w.w_std, w.seed, _S_W_UV)
    return w_uk, w_uv


def cache_raw(w: Workload, b: int, n_tokens: int):
    """Raw draws for sequence b's first n_tokens cache rows.

    Returns (c_raw [n, d_c], pe_raw [n, d_r]) fp32 N(0,1). Whether they are
    stored as-is or first normalised/rotated is the caller's business
    (see ``Workload.kv_values``).
    """
    d = w.dims
    t = normal((n_tokens, d.row_width), 1.0, w.seed, _S_CACHE + b)
    return t[:, : d.kv_lora_rank], t[:, d.kv_lora_rank:]


def append_inputs(w: Workload):
    """Inputs of the cache append for workloads that have one.

    x [B*Sq, hidden] ~ N(0,1) hidden states of the newest tokens, W_kva
    [hidden, d_c + d_r] ~ N(0, append_w_std^2), and the (sequence, position)
    of every new token: sequence b's new tokens sit at positions
    L_b - Sq .. L_b - 1.
    """
    if not w.append_hidden:
        return None
    d = w.dims
    lengths = context_lengths(w)
    n = w.batch * w.q_len
    x = normal((n, w.append_hidden), 1.0, w.seed, _S_X)
    w_kva = normal((w.append_hidden, d.row_width), w.append_w_std, w.seed, _S_W_KVA)
    seq_ids = torch.arange(w.batch, dtype=torch.int32).repeat_interleave(w.q_len)
    offs = torch.arange(w.q_len, dtype=torch.int32).repeat(w.batch)
    positions = lengths.repeat_interleave(w.q_len) - w.q_len + offs
    return dict(x=x, w_kva=w_kva, seq_ids=seq_ids, positions=positions.to(torch.int32))


def q_proj_inputs(dims: Dims, n_tokens: int, hidden: int, q_rank: int, seed: int, gamma: bool = True,
                  max_position: int = 32768):
    """bf16 inputs of the query projection: x [T, hidden] ~ N(0,1), W_qa
    [hidden, q_rank] ~ N(0, 1/hidden), W_qb [q_rank, H (d_n + d_r)] ~
    N(0, 1/q_rank), gamma [q_rank] ~ U[0.5, 1.5] (or None) and positions
    int32 [T] ~ U[0, max_position)."""
    x = bf16(normal((n_tokens, hidden), 1.0, seed, _S_QX))
    w_qa = bf16(normal((hidden, q_rank), hidden ** -0.5, seed, _S_W_QA))
    n2 = dims.num_heads * (dims.qk_nope_dim + dims.rope_dim)
    w_qb = bf16(normal((q_rank, n2), q_rank ** -0.5, seed, _S_W_QB))
    g = None
    if gamma:
        g = bf16(0.5 + torch.rand(q_rank, generator=generator(seed, _S_QGAMMA)))
    pos = torch.randint(0, max_position, (n_tokens,), generator=generator(seed, _S_QPOS), dtype=torch.int32)
    return dict(x=x, w_qa=w_qa, w_qb=w_qb, gamma=g, positions=pos)


def scaled(w: Workload, batch: Optional[int] = None, length: Optional[int] = None,
           q_len: Optional[int] = None, name: Optional[str] = None, **kw) -> Workload:
    """A smaller copy of a workload (same dims and value recipe)."""
    rng = w.length_range if length is None else (length, length)
    return dataclasses.replace(
        w, name=name or (w.name + "_scaled"), batch=w.batch if batch is None else batch,
        q_len=w.q_len if q_len is None else q_len, length_range=rng, **kw)
