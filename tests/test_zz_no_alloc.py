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
    from mla_latent_kv_29_b200 import lib as L

    lib = L.load()
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    cd = L.c_dims(w.dims, w.softmax_scale)
    assert lib.mla_decode_workspace_size(ctypes.byref(cd), 64, 1, 8192, None) <= L.NO_ALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)  # never touched: the size check comes first
    rc = lib.mla_decode_no_alloc(ctypes.byref(cd), fake, fake, 4096, 1, fake, 100, fake, 128, fake, 8192, fake,
                                 fake, fake, None, None)
    assert rc == -8
    assert "scratch" in L.error_string(rc)
