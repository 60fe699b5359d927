"""ctypes binding of libmla_b200.so (argument marshalling only).

Each function mirrors the C entry point of the same name in
``include/mla_b200.h``: it checks tensor dtypes/shapes/devices, passes raw
device pointers and the current CUDA stream, and raises ``MLAError`` on a
non-zero status. Torch is used for device memory and streams only; every
step of the computation runs in the library's kernels. There is no CPU path:
without the built library or a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .inputs import Dims

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200.so")

MLA_OK = 0
STATUS_NAMES = {
    0: "MLA_OK", -1: "MLA_ERR_INVALID_ARG", -2: "MLA_ERR_UNSUPPORTED_DIMS",
    -3: "MLA_ERR_WORKSPACE_TOO_SMALL", -4: "MLA_ERR_CUDA", -5: "MLA_ERR_DEVICE_FAULT",
    -6: "MLA_ERR_DEVICE_TIMEOUT", -7: "MLA_ERR_NO_DEVICE", -8: "MLA_ERR_SCRATCH_LIMIT",
}
NO_ALLOC_SCRATCH_BYTES = 48 * 1024 * 1024  # MLA_NO_ALLOC_SCRATCH_BYTES
KERNEL_AUTO, KERNEL_SM100, KERNEL_GENERIC = 0, 1, 2

EXPORTED = ("mla_append_kv", "mla_append_workspace_size", "mla_decode", "mla_decode_workspace_size",
            "mla_combine", "mla_debug_resolve_slots", "mla_get_device_error", "mla_error_string",
            "mla_version", "mla_decode_no_alloc", "mla_q_proj", "mla_q_proj_workspace_size", "mla_o_proj",
            "mla_o_proj_workspace_size", "mla_append_kv_fp8", "mla_cache_to_fp8", "mla_fp8_block_bytes")


class MLAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({error_string(status)})")


class CDims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("kv_lora_rank", ctypes.c_int32), ("rope_dim", ctypes.c_int32),
                ("qk_nope_dim", ctypes.c_int32), ("v_head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class CDecodeOpts(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("num_workers", ctypes.c_int32),
                ("event_attn_begin", ctypes.c_void_p), ("event_attn_end", ctypes.c_void_p),
                ("cache_ready", ctypes.c_void_p), ("debug_wait_limit_us", ctypes.c_uint32),
                ("debug_starve", ctypes.c_int32), ("output_latent", ctypes.c_int32), ("cache_fp8", ctypes.c_int32)]


_lib = None
_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float


def load():
    """Loads the library once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mla_latent_kv_29_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    D = ctypes.POINTER(CDims)
    O = ctypes.POINTER(CDecodeOpts)
    sig = {
        "mla_append_kv": (_I32, [D, _P, _I32, _I32, _P, _P, _F, _F, _P, _P, _P, _I32, _I32, _P, _I64, _P, _SZ, _P]),
        "mla_append_workspace_size": (_SZ, [D, _I32, _I32]),
        "mla_decode": (_I32, [D, _P, _P, _I32, _I32, _P, _I64, _P, _I32, _P, _I32, _P, _P, _P, _P, _SZ, O, _P]),
        "mla_decode_workspace_size": (_SZ, [D, _I32, _I32, _I32, O]),
        "mla_combine": (_I32, [D, _P, _P, _P, _I32, _P, _P, _P]),
        "mla_debug_resolve_slots": (_I32, [D, _P, _I32, _I32, _I64, _P, _P, _I32, _P, _P]),
        "mla_get_device_error": (_I32, [ctypes.POINTER(ctypes.c_int), _P]),
        "mla_error_string": (ctypes.c_char_p, [_I32]),
        "mla_version": (_I32, []),
        "mla_decode_no_alloc": (_I32, [D, _P, _P, _I32, _I32, _P, _I64, _P, _I32, _P, _I32, _P, _P, _P, O, _P]),
        "mla_q_proj": (_I32, [D, _P, _I32, _I32, _P, _I32, _P, _F, _P, _P, _F, _P, _P, _P, _SZ, _P]),
        "mla_q_proj_workspace_size": (_SZ, [D, _I32, _I32, _I32]),
        "mla_o_proj": (_I32, [_P, _I32, _I32, _P, _I32, _P, _P, _SZ, _P]),
        "mla_o_proj_workspace_size": (_SZ, [_I32, _I32, _I32]),
        "mla_append_kv_fp8": (_I32, [D, _P, _I32, _I32, _P, _P, _F, _F, _P, _P, _P, _I32, _I32, _P, _I64, _P, _SZ, _P]),
        "mla_cache_to_fp8": (_I32, [D, _P, _I64, _P, _P]),
        "mla_fp8_block_bytes": (_SZ, [D]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def error_string(status: int) -> str:
    return load().mla_error_string(int(status)).decode()


def c_dims(d: Dims, softmax_scale: float) -> CDims:
    return CDims(d.num_heads, d.kv_lora_rank, d.rope_dim, d.qk_nope_dim, d.v_head_dim, d.block_size,
                 float(softmax_scale))


def _event_handle(ev) -> Optional[int]:
    # torch creates the CUDA event on its first record(); make sure the handle exists
    if ev.cuda_event == 0:
        ev.record()
    return ev.cuda_event


def c_opts(kernel: int = KERNEL_AUTO, num_workers: int = 0, events=None, cache_ready=None,
           debug_wait_limit_us: int = 0, debug_starve: bool = False, output_latent: bool = False,
           cache_fp8: bool = False) -> CDecodeOpts:
    b, e = (None, None) if events is None else (_event_handle(events[0]), _event_handle(events[1]))
    r = None if cache_ready is None else _event_handle(cache_ready)
    return CDecodeOpts(int(kernel), int(num_workers), b, e, r, int(debug_wait_limit_us), int(bool(debug_starve)),
                       int(bool(output_latent)), int(bool(cache_fp8)))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(None)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int, what: str):
    if status != MLA_OK:
        raise MLAError(status, what)


_nvtx = False


def set_nvtx(on: bool = True) -> None:
    """Mark every library call with an NVTX range named after its C entry point
    (visible in Nsight timelines); off by default, which costs nothing."""
    global _nvtx
    _nvtx = bool(on)


def _call(name: str, *args) -> int:
    """Calls C entry point `name`, inside an NVTX range of that name when enabled."""
    fn = getattr(load(), name)
    if not _nvtx:
        return fn(*args)
    torch.cuda.nvtx.range_push(name)
    try:
        return fn(*args)
    finally:
        torch.cuda.nvtx.range_pop()


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ append
def append_workspace_size(dims: Dims, n_tokens: int, hidden: int, softmax_scale: float = 1.0) -> int:
    return int(load().mla_append_workspace_size(ctypes.byref(c_dims(dims, softmax_scale)), n_tokens, hidden))


def append_kv(dims: Dims, x, w_kva, seq_ids, positions, block_table, pool, rms_gamma=None,
              rms_eps: float = 1e-6, rope_base: float = 10000.0, workspace=None, stream=None, fp8: bool = False):
    """mla_append_kv into a bf16 pool, or (fp8) mla_append_kv_fp8 into an FP8 pool
    (uint8 [num_blocks, fp8_block_bytes(dims)])."""
    lib = load()
    cd = c_dims(dims, 1.0)
    T, hidden = x.shape
    need = lib.mla_append_workspace_size(ctypes.byref(cd), T, hidden)
    if workspace is None:
        workspace = _workspace(need, x.device)
    name = "mla_append_kv_fp8" if fp8 else "mla_append_kv"
    st = _call(
        name, ctypes.byref(cd), _ptr(x, torch.bfloat16, "x"), T, hidden, _ptr(w_kva, torch.bfloat16, "w_kva"),
        _ptr(rms_gamma, torch.bfloat16, "rms_gamma"), float(rms_eps), float(rope_base),
        _ptr(seq_ids, torch.int32, "seq_ids"), _ptr(positions, torch.int32, "positions"),
        _ptr(block_table, torch.int32, "block_table"), block_table.shape[0], block_table.shape[1],
        _ptr(pool, torch.uint8 if fp8 else torch.bfloat16, "pool"), pool.shape[0], _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, name)
    return pool


# ---------------------------------------------------------------- FP8 cache
def fp8_block_bytes(dims: Dims) -> int:
    return int(load().mla_fp8_block_bytes(ctypes.byref(c_dims(dims, 1.0))))


def cache_to_fp8(dims: Dims, pool, out=None, stream=None):
    """mla_cache_to_fp8: the FP8 pool (uint8 [num_blocks, fp8_block_bytes]) of a bf16 pool."""
    lib = load()
    nb = pool.shape[0]
    bb = fp8_block_bytes(dims)
    if bb == 0:
        raise MLAError(-2, "mla_fp8_block_bytes")
    if out is None:
        out = torch.empty(nb, bb, dtype=torch.uint8, device=pool.device)
    st = _call("mla_cache_to_fp8", ctypes.byref(c_dims(dims, 1.0)), _ptr(pool, torch.bfloat16, "pool"), nb,
                              _ptr(out, torch.uint8, "pool_fp8"), _stream(stream))
    _check(st, "mla_cache_to_fp8")
    return out


# -------------------------------------------------------- query projection
def q_proj_workspace_size(dims: Dims, n_tokens: int, hidden: int, q_rank: int) -> int:
    return int(load().mla_q_proj_workspace_size(ctypes.byref(c_dims(dims, 1.0)), n_tokens, hidden, q_rank))


def q_proj(dims: Dims, x, w_qa, w_qb, positions, q_gamma=None, rms_eps: float = 1e-6, rope_base: float = 10000.0,
           q_nope=None, q_pe=None, workspace=None, stream=None):
    """mla_q_proj: (q_nope [T, H, d_n], q_pe [T, H, d_r]) bf16 from x [T, hidden]."""
    lib = load()
    cd = c_dims(dims, 1.0)
    T, hidden = x.shape
    q_rank = w_qa.shape[1]
    need = lib.mla_q_proj_workspace_size(ctypes.byref(cd), T, hidden, q_rank)
    if need == 0:
        raise MLAError(-2, "mla_q_proj_workspace_size")
    if workspace is None:
        workspace = _workspace(need, x.device)
    if q_nope is None:
        q_nope = torch.empty(T, dims.num_heads, dims.qk_nope_dim, dtype=torch.bfloat16, device=x.device)
    if q_pe is None:
        q_pe = torch.empty(T, dims.num_heads, dims.rope_dim, dtype=torch.bfloat16, device=x.device)
    st = _call("mla_q_proj",
        ctypes.byref(cd), _ptr(x, torch.bfloat16, "x"), T, hidden, _ptr(w_qa, torch.bfloat16, "w_qa"), q_rank,
        _ptr(q_gamma, torch.bfloat16, "q_gamma"), float(rms_eps), _ptr(w_qb, torch.bfloat16, "w_qb"),
        _ptr(positions, torch.int32, "positions"), float(rope_base), _ptr(q_nope, torch.bfloat16, "q_nope"),
        _ptr(q_pe, torch.bfloat16, "q_pe"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "mla_q_proj")
    return q_nope, q_pe


# ------------------------------------------------------- output projection
def o_proj_workspace_size(n_tokens: int, k: int, n: int) -> int:
    return int(load().mla_o_proj_workspace_size(n_tokens, k, n))


def o_proj(x, w, y=None, workspace=None, stream=None):
    """mla_o_proj: y [T, n] = bf16(x [T, k] . w [k, n]); x may be any contiguous
    tensor whose trailing dims flatten to k (e.g. the decode output [B, Sq, H, d_v])."""
    lib = load()
    x2 = x.reshape(-1, w.shape[0]) if x.dim() != 2 else x
    T, k = x2.shape
    n = w.shape[1]
    need = lib.mla_o_proj_workspace_size(T, k, n)
    if need == 0:
        raise MLAError(-2, "mla_o_proj_workspace_size")
    if workspace is None:
        workspace = _workspace(need, x.device)
    if y is None:
        y = torch.empty(T, n, dtype=torch.bfloat16, device=x.device)
    st = _call("mla_o_proj", _ptr(x2, torch.bfloat16, "x"), T, k, _ptr(w, torch.bfloat16, "w"), n,
                        _ptr(y, torch.bfloat16, "y"), _ptr(workspace, None, "workspace"),
                        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "mla_o_proj")
    return y


# ------------------------------------------------------------------ decode
def decode_workspace_size(dims: Dims, softmax_scale: float, batch: int, q_len: int, max_context_len: int,
                          kernel: int = KERNEL_AUTO, num_workers: int = 0) -> int:
    o = c_opts(kernel, num_workers)
    return int(load().mla_decode_workspace_size(ctypes.byref(c_dims(dims, softmax_scale)), batch, q_len,
                                                 max_context_len, ctypes.byref(o)))


def decode(dims: Dims, softmax_scale: float, q_nope, q_pe, pool, block_table, context_lens,
           max_context_len: int, w_uk, w_uv, out=None, workspace=None, kernel: int = KERNEL_AUTO,
           num_workers: int = 0, stream=None, attn_events=None, cache_ready=None, debug_wait_limit_us: int = 0,
           debug_starve: bool = False, output_latent: bool = False, cache_fp8: bool = False):
    """attn_events: optional (begin, end) torch.cuda.Event pair recorded around the
    attention kernel on the launch stream. cache_ready: optional torch.cuda.Event
    (already recorded once, so that it has a handle) that the attention launch
    waits for, e.g. recorded after an append_kv on another stream.
    debug_wait_limit_us / debug_starve: the failure-detection test hooks of
    mla_decode_opts_t (leave at 0 / False). output_latent: return o_lat
    [B, Sq, H, d_c] instead of the up-projected output (w_uv is not read).
    cache_fp8: `pool` is an FP8 pool (uint8 [num_blocks, fp8_block_bytes])."""
    lib = load()
    cd = c_dims(dims, softmax_scale)
    o = c_opts(kernel, num_workers, attn_events, cache_ready, debug_wait_limit_us, debug_starve, output_latent,
               cache_fp8)
    B, Sq = q_nope.shape[0], q_nope.shape[1]
    if out is None:
        width = dims.kv_lora_rank if output_latent else dims.v_head_dim
        out = torch.empty(B, Sq, dims.num_heads, width, dtype=torch.bfloat16, device=q_nope.device)
    need = lib.mla_decode_workspace_size(ctypes.byref(cd), B, Sq, int(max_context_len), ctypes.byref(o))
    if need == 0:
        raise MLAError(-2, "mla_decode_workspace_size")
    if workspace is None:
        workspace = _workspace(need, q_nope.device)
    st = _call("mla_decode",
        ctypes.byref(cd), _ptr(q_nope, torch.bfloat16, "q_nope"), _ptr(q_pe, torch.bfloat16, "q_pe"), B, Sq,
        _ptr(pool, torch.uint8 if cache_fp8 else torch.bfloat16, "pool"), pool.shape[0],
        _ptr(block_table, torch.int32, "block_table"),
        block_table.shape[1], _ptr(context_lens, torch.int32, "context_lens"), int(max_context_len),
        _ptr(w_uk, torch.bfloat16, "w_uk"), _ptr(w_uv, torch.bfloat16, "w_uv"),
        _ptr(out, torch.bfloat16, "out"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), ctypes.byref(o), _stream(stream))
    _check(st, "mla_decode")
    return out


def decode_no_alloc(dims: Dims, softmax_scale: float, q_nope, q_pe, pool, block_table, context_lens,
                    max_context_len: int, w_uk, w_uv, out=None, kernel: int = KERNEL_AUTO, num_workers: int = 0,
                    stream=None, cache_fp8: bool = False):
    """mla_decode with the library's built-in scratch buffer (no workspace argument)."""
    lib = load()
    cd = c_dims(dims, softmax_scale)
    o = c_opts(kernel, num_workers, cache_fp8=cache_fp8)
    B, Sq = q_nope.shape[0], q_nope.shape[1]
    if out is None:
        out = torch.empty(B, Sq, dims.num_heads, dims.v_head_dim, dtype=torch.bfloat16, device=q_nope.device)
    st = _call("mla_decode_no_alloc",
        ctypes.byref(cd), _ptr(q_nope, torch.bfloat16, "q_nope"), _ptr(q_pe, torch.bfloat16, "q_pe"), B, Sq,
        _ptr(pool, torch.uint8 if cache_fp8 else torch.bfloat16, "pool"), pool.shape[0],
        _ptr(block_table, torch.int32, "block_table"),
        block_table.shape[1], _ptr(context_lens, torch.int32, "context_lens"), int(max_context_len),
        _ptr(w_uk, torch.bfloat16, "w_uk"), _ptr(w_uv, torch.bfloat16, "w_uv"),
        _ptr(out, torch.bfloat16, "out"), ctypes.byref(o), _stream(stream))
    _check(st, "mla_decode_no_alloc")
    return out


# ----------------------------------------------------------------- combine
def combine(dims: Dims, o_part, lse_part, part_offsets, o_lat=None, lse_out=None, stream=None):
    lib = load()
    cd = c_dims(dims, 1.0)
    G = part_offsets.numel() - 1
    if o_lat is None:
        o_lat = torch.empty(G, dims.num_heads, dims.kv_lora_rank, dtype=torch.float32, device=o_part.device)
    st = _call("mla_combine", ctypes.byref(cd), _ptr(o_part, torch.float32, "o_part"),
                         _ptr(lse_part, torch.float32, "lse_part"), _ptr(part_offsets, torch.int32, "part_offsets"),
                         G, _ptr(o_lat, torch.float32, "o_lat"), _ptr(lse_out, torch.float32, "lse_out"),
                         _stream(stream))
    _check(st, "mla_combine")
    return o_lat


# ------------------------------------------------------------------- debug
def resolve_slots(dims: Dims, block_table, num_blocks: int, seq_ids, positions, stream=None):
    lib = load()
    rows = torch.empty(seq_ids.numel(), dtype=torch.int64, device=seq_ids.device)
    st = lib.mla_debug_resolve_slots(ctypes.byref(c_dims(dims, 1.0)), _ptr(block_table, torch.int32, "block_table"),
                                     block_table.shape[0], block_table.shape[1], int(num_blocks),
                                     _ptr(seq_ids, torch.int32, "seq_ids"), _ptr(positions, torch.int32, "positions"),
                                     seq_ids.numel(), _ptr(rows, torch.int64, "rows"), _stream(stream))
    _check(st, "mla_debug_resolve_slots")
    return rows


def device_error(stream=None) -> int:
    v = ctypes.c_int(0)
    _check(load().mla_get_device_error(ctypes.byref(v), _stream(stream)), "mla_get_device_error")
    return v.value
