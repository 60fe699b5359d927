"""mla_decode_no_alloc: decode for callers that cannot allocate device memory
(a plugin inside a host process that owns all device memory, a path that
cannot afford cudaMalloc's synchronisation, plain C without a memory
manager). Its scratch is a fixed buffer compiled into the library, so the
test checks, through the C ABI, that two calls in a row -- on different
problems, sharing that buffer -- match the allocating mla_decode within the
decode tolerance, and that a problem too large for the buffer is refused
before any work is enqueued. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from mla_latent_kv_29_b200 import inputs as I

from _data import build, to_device, tolerance_ok

pytestmark = pytest.mark.gpu


def _case(name, batch, q_len, lengths):
    w = I.scaled(I.WORKLOADS["v3_b64_l1k_8k"], batch=batch, q_len=q_len, name=name)
    data = build(w, lengths=torch.tensor(lengths, dtype=torch.int32))
    return w, to_device(data)


def _decode_pair(L, w, dd):
    args = (w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], dd["pool"], dd["table"], dd["lengths"],
            int(dd["lengths"].max()), dd["w_uk"], dd["w_uv"])
    ref = L.decode(*args)
    got = L.decode_no_alloc(*args)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return got.float().cpu().numpy(), ref.float().cpu().numpy()


def test_no_alloc_matches_decode_on_two_calls_in_a_row():
    from mla_latent_kv_29_b200 import lib as L

    L.load()
    first = _case("no_alloc_a", 3, 2, [70, 129, 300])
    second = _case("no_alloc_b", 5, 1, [1, 64, 65, 1000, 257])
    for w, dd in (first, second):
        got, ref = _decode_pair(L, w, dd)
        assert np.all(np.isfinite(got))
        ok, err, bound = tolerance_ok(got, ref)
        assert ok, f"max|err| {err:.3e} > {bound:.3e}"


def test_no_alloc_refuses_problems_beyond_its_buffer():
    """Batch 128 with one-token contexts needs more scratch than the buffer
    holds (the absorbed queries and the split partials grow with the batch):
    the call returns MLA_ERR_SCRATCH_LIMIT and leaves the output untouched.
    Every argument is a real device tensor of the stated shape."""
    from mla_latent_kv_29_b200 import lib as L

    lib = L.load()
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    d = w.dims
    cd = L.c_dims(d, w.softmax_scale)
    B = 128
    assert lib.mla_decode_workspace_size(ctypes.byref(cd), 64, 1, 8192, None) <= L.NO_ALLOC_SCRATCH_BYTES
    assert lib.mla_decode_workspace_size(ctypes.byref(cd), B, 1, 1, None) > L.NO_ALLOC_SCRATCH_BYTES
    dev = "cuda"
    q_nope = torch.zeros(B, 1, d.num_heads, d.qk_nope_dim, dtype=torch.bfloat16, device=dev)
    q_pe = torch.zeros(B, 1, d.num_heads, d.rope_dim, dtype=torch.bfloat16, device=dev)
    pool = torch.zeros(B, d.block_size, d.row_width, dtype=torch.bfloat16, device=dev)
    table = torch.arange(B, dtype=torch.int32, device=dev).view(B, 1)
    lengths = torch.ones(B, dtype=torch.int32, device=dev)
    w_uk = torch.zeros(d.num_heads, d.qk_nope_dim, d.kv_lora_rank, dtype=torch.bfloat16, device=dev)
    w_uv = torch.zeros(d.num_heads, d.v_head_dim, d.kv_lora_rank, dtype=torch.bfloat16, device=dev)
    out = torch.full((B, 1, d.num_heads, d.v_head_dim), 7.0, dtype=torch.bfloat16, device=dev)
    with pytest.raises(L.MLAError) as e:
        L.decode_no_alloc(d, w.softmax_scale, q_nope, q_pe, pool, table, lengths, 1, w_uk, w_uv, out=out)
    assert e.value.status == -8
    assert "scratch" in L.error_string(e.value.status)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert bool(torch.all(out == 7.0))  # nothing was enqueued
