"""Builds concrete test inputs from the seeded generators.

Cache rows of "rmsnorm_rope" workloads are the raw N(0,1) draws passed
through the oracle's RMSNorm (latent part) and RoPE at the token position
(RoPE part), then stored as bf16. The GPU and the oracle both read the same
bf16 pool. Nothing here reads a value computed by the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_29_b200 import inputs as I
from oracle import mla_oracle as O


def token_rows(table: np.ndarray, b: int, n: int, bs: int) -> np.ndarray:
    t = np.arange(n)
    return table[b, t // bs].astype(np.int64) * bs + t % bs


def cache_rows(w: I.Workload, b: int, n: int) -> torch.Tensor:
    """bf16 [n, d_c + d_r] rows of sequence b's first n tokens."""
    c_raw, pe_raw = I.cache_raw(w, b, n)
    if w.kv_values == "rmsnorm_rope":
        c = O.rmsnorm(c_raw)
        pe = O.rope(pe_raw, np.arange(n))
        return torch.from_numpy(np.concatenate([c, pe], axis=1)).to(torch.bfloat16)
    return torch.cat([c_raw, pe_raw], dim=1).to(torch.bfloat16)


def build(w: I.Workload, fill: float = 0.0, lengths=None):
    """Host (CPU) tensors of a decode workload.

    The pool holds every cached token; for workloads with an append, the
    q_len newest tokens of each sequence are NOT in the pool (their rows are
    left at ``fill``) and the append inputs are returned instead.
    """
    d = w.dims
    if lengths is None:
        lengths = I.context_lengths(w)
    lengths = lengths.to(torch.int32)
    table, nblocks = I.block_table(w, lengths)
    pool = torch.full((nblocks, d.block_size, d.row_width), fill, dtype=torch.bfloat16)
    flat = pool.view(-1, d.row_width)
    tab = table.numpy()
    n_new = w.q_len if w.append_hidden else 0
    for b, L in enumerate(lengths.tolist()):
        n = L - n_new
        if n > 0:
            flat[torch.from_numpy(token_rows(tab, b, n, d.block_size))] = cache_rows(w, b, n)
    q_nope, q_pe = I.queries(w)
    w_uk, w_uv = I.up_weights(w)
    out = dict(lengths=lengths, table=table, num_blocks=nblocks, pool=pool,
               q_nope=I.bf16(q_nope), q_pe=I.bf16(q_pe), w_uk=I.bf16(w_uk), w_uv=I.bf16(w_uv))
    ap = I.append_inputs(w) if w.append_hidden else None
    if ap is not None:
        out["append"] = dict(x=I.bf16(ap["x"]), w_kva=I.bf16(ap["w_kva"]), seq_ids=ap["seq_ids"],
                             positions=ap["positions"])
    return out


def oracle_append_pool(w: I.Workload, data) -> torch.Tensor:
    """The pool after the oracle's append (rows rounded to bf16 storage)."""
    d = w.dims
    ap = data["append"]
    rows = O.append_rows(ap["x"], ap["w_kva"], ap["positions"].numpy(), d.kv_lora_rank)
    pool = data["pool"].clone()
    flat = pool.view(-1, d.row_width)
    tab = data["table"].numpy()
    slots = [O.resolve_slot(tab, int(b), int(p), d.block_size)
             for b, p in zip(ap["seq_ids"].tolist(), ap["positions"].tolist())]
    flat[torch.tensor(slots)] = torch.from_numpy(rows).to(torch.bfloat16)
    return pool


def to_device(data, device="cuda"):
    out = {}
    for k, v in data.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.to(device)
        elif isinstance(v, dict):
            out[k] = to_device(v, device)
        else:
            out[k] = v
    return out


def tolerance_ok(got: np.ndarray, ref: np.ndarray):
    """max|err| <= 2e-2 * max|ref| + 1e-3 over the compared entries."""
    err = float(np.max(np.abs(got - ref)))
    bound = 2e-2 * float(np.max(np.abs(ref))) + 1e-3
    return err <= bound, err, bound
