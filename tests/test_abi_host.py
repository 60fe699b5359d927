"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before touching a device. No kernel is
launched here; on a machine without a GPU a fully valid call must return
MLA_ERR_NO_DEVICE rather than crash."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_29_b200 import inputs as I
from mla_latent_kv_29_b200 import lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def so():
    if not os.path.exists(L.LIB_PATH):
        from mla_latent_kv_29_b200 import build

        build.build()
    return L.load()


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(so):
    names = declared_symbols()
    assert {"mla_append_kv", "mla_decode", "mla_combine"} <= names
    for n in names:
        assert hasattr(so, n), n
    assert set(L.EXPORTED) == names


def test_error_strings_and_version(so):
    for code in L.STATUS_NAMES:
        assert L.error_string(code)
    assert L.error_string(12345) == "unknown status"
    assert so.mla_version() >= 100


def _dims(**kw):
    d = dict(num_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope_dim=128, v_head_dim=128, block_size=64,
             softmax_scale=192 ** -0.5)
    d.update(kw)
    return L.CDims(**d)


def _decode(so, dims, ws_bytes=1 << 30, null_q=False, batch=2, q_len=1, max_len=1000, opts=None):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first or no device
    return so.mla_decode(ctypes.byref(dims), None if null_q else fake, fake, batch, q_len, fake, 100, fake, 16,
                         fake, max_len, fake, fake, fake, ctypes.c_void_p(1 << 20), ws_bytes,
                         ctypes.byref(opts) if opts else None, None)


def test_workspace_size_v3(so):
    n = so.mla_decode_workspace_size(ctypes.byref(_dims()), 64, 1, 8192, None)
    assert n > 64 * 128 * 576 * 2  # at least the absorbed queries
    assert n % 256 == 0
    assert so.mla_decode_workspace_size(ctypes.byref(_dims(num_heads=0)), 64, 1, 8192, None) == 0
    assert so.mla_decode_workspace_size(ctypes.byref(_dims()), 4, 8, 4, None) == 0  # max_len < q_len
    assert so.mla_append_workspace_size(ctypes.byref(_dims()), 64, 7168) >= 64 * 576 * 4


def test_decode_validation(so):
    assert _decode(so, _dims(), null_q=True) == -1
    assert _decode(so, _dims(kv_lora_rank=4096)) == -2
    assert _decode(so, _dims(rope_dim=3)) == -1 or _decode(so, _dims(rope_dim=3)) == -2
    assert _decode(so, _dims(softmax_scale=float("nan"))) == -1
    assert _decode(so, _dims(), ws_bytes=16) == -3
    assert _decode(so, _dims(), batch=0) == -1
    assert _decode(so, _dims(), max_len=2000) == -1  # 16 pages of 64 do not cover 2000 tokens


def test_combine_and_append_validation(so):
    d = _dims()
    assert so.mla_combine(ctypes.byref(d), None, None, None, 4, None, None, None) == -1
    fake = ctypes.c_void_p(1 << 20)
    assert so.mla_append_kv(ctypes.byref(d), fake, 0, 7168, fake, None, 1e-6, 1e4, fake, fake, fake, 16, 1, fake,
                            10, fake, 1 << 30, None) == -1
    assert so.mla_append_kv(ctypes.byref(d), fake, 64, 7168, fake, None, 1e-6, 1e4, fake, fake, fake, 16, 1, fake,
                            10, fake, 16, None) == -3


def test_q_proj_validation(so):
    d = _dims()
    ws = so.mla_q_proj_workspace_size(ctypes.byref(d), 64, 7168, 1536)
    # GEMM 1 partials (fp32 T x q_rank), c_q (bf16), GEMM 2 partials (fp32 T x H * 192)
    assert ws >= 64 * 1536 * 4 + 64 * 1536 * 2 + 64 * 128 * 192 * 4 and ws % 256 == 0
    assert so.mla_q_proj_workspace_size(ctypes.byref(d), 64, 7000, 1536) == 0  # hidden not a multiple of 64
    assert so.mla_q_proj_workspace_size(ctypes.byref(d), 0, 7168, 1536) == 0
    fake = ctypes.c_void_p(1 << 20)

    def call(T=64, hidden=7168, rank=1536, x=fake, ws_bytes=1 << 30, eps=1e-6):
        return so.mla_q_proj(ctypes.byref(d), x, T, hidden, fake, rank, None, eps, fake, fake, 1e4, fake, fake,
                             fake, ws_bytes, None)

    assert call(x=None) == -1
    assert call(T=0) == -1
    assert call(hidden=7000) == -2
    assert call(eps=-1.0) == -1
    assert call(ws_bytes=16) == -3


def test_fp8_cache_validation(so):
    d = _dims()
    assert so.mla_fp8_block_bytes(ctypes.byref(d)) == 64 * 640 + 256  # 41216: 644 bytes per token
    assert so.mla_fp8_block_bytes(ctypes.byref(_dims(kv_lora_rank=520))) == 0  # latent not a multiple of 16
    assert so.mla_fp8_block_bytes(ctypes.byref(_dims(block_size=62))) == 0  # scales not 16-byte aligned
    fake = ctypes.c_void_p(1 << 20)
    assert so.mla_cache_to_fp8(ctypes.byref(d), None, 10, fake, None) == -1
    assert so.mla_cache_to_fp8(ctypes.byref(d), fake, 0, fake, None) == -1
    assert so.mla_cache_to_fp8(ctypes.byref(d), ctypes.c_void_p((1 << 20) + 8), 10, fake, None) == -1  # unaligned
    assert so.mla_cache_to_fp8(ctypes.byref(_dims(rope_dim=4)), fake, 10, fake, None) == -2
    assert so.mla_append_kv_fp8(ctypes.byref(_dims(rope_dim=4)), fake, 64, 7168, fake, None, 1e-6, 1e4, fake, fake,
                                fake, 16, 1, fake, 10, fake, 1 << 30, None) == -2
    assert so.mla_append_kv_fp8(ctypes.byref(d), fake, 64, 7168, fake, None, 1e-6, 1e4, fake, fake, fake, 16, 1,
                                fake, 10, fake, 16, None) == -3
    # an FP8 decode needs the tensor-core kernel: the CUDA-core kernel refuses it before any launch
    opts = L.c_opts(kernel=2, cache_fp8=True)
    assert _decode(so, d, opts=opts) == -2


def test_valid_call_without_gpu_reports_no_device(so):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _decode(so, _dims()) == -7
    assert so.mla_combine(ctypes.byref(_dims()), ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 20),
                          ctypes.c_void_p(1 << 20), 4, ctypes.c_void_p(1 << 20), None, None) == -7


def test_python_binding_has_no_cpu_path():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    w = I.WORKLOADS["tiny_b1_l128"]
    q = torch.zeros(1, 1, 16, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        L.decode(w.dims, w.softmax_scale, q, q, q, q, q, 128, q, q)


def test_nvtx_ranges_wrap_the_calls(monkeypatch):
    """With NVTX on, each entry point runs inside a range of its own name, and the
    range is closed even when the call fails."""
    import torch

    pushed, popped = [], []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda n: pushed.append(n))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: popped.append(1))
    L.set_nvtx(True)
    try:
        st = L._call("mla_combine", ctypes.byref(_dims()), None, None, None, 4, None, None, None)
    finally:
        L.set_nvtx(False)
    assert st == -1 and pushed == ["mla_combine"] and len(popped) == 1
    L._call("mla_combine", ctypes.byref(_dims()), None, None, None, 4, None, None, None)
    assert pushed == ["mla_combine"]  # off again: no range
