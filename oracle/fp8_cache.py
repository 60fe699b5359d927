"""fp64 CPU oracle of the FP8 (e4m3) latent cache.

TEST INFRASTRUCTURE ONLY, like ``mla_oracle``: only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the library never does, and the two share no code.

Source: [MLA-arch] "MLA架构：低秩注意力机制优化LLM显存与计算效率", section 4.2,
item 3 ("量化的影响"): quantising the cache shrinks it further, with a
warning about numerical stability. The page names no format, so this module
fixes one (a reading, stated here and in the library header):

* values: OCP 8-bit floating point E4M3 ("fn" variant): 1 sign bit, 4
  exponent bits with bias 7, 3 mantissa bits; exponent field 0 is
  subnormal (m * 2^-9); S.1111.111 is NaN; no infinities; the largest
  finite magnitude is 448. Encoding rounds to nearest, ties to the even
  code, and saturates to +-448.
* scale: one power of two per token, s_t = 2^e_t with e_t the smallest
  integer such that amax_t <= 448 * 2^e_t (amax_t = max |c_t| over the
  token's latent values), clamped to [-15, 7]. Dividing by a power of two
  is exact, so the only rounding is the e4m3 one, and every dequantised
  value code * 2^e is exactly an IEEE half (f16) for e in that range.
* RoPE key: stored as f16 (rounded to nearest even), not quantised: it is
  8 % of the row and carries the position signal.
* layout of one cache block of ``block_size`` tokens: block_size rows of
  d_c + 2 d_r bytes (d_c e4m3 codes, then d_r f16 little-endian), followed
  by block_size fp32 scales s_t. For DeepSeek-V3 dims a block is
  64 * 640 + 256 = 41216 bytes: 644 bytes per token against 1152 for bf16.
* the dequantised cache is c~_t = decode(code) * s_t and k~_pe = f16 value;
  attention over the FP8 cache is the fp64 definition of ``mla_oracle``
  applied to the dequantised cache.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN = 0x7F
SCALE_EXP_MIN, SCALE_EXP_MAX = -15, 7


def e4m3_value(code: int) -> float:
    """Value of one e4m3 code, from the field definition (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """float64 [256]: the value of every code."""
    return np.array([e4m3_value(c) for c in range(256)])


def _positive_grid():
    """Codes 0x00..0x7E (the non-negative finite values, increasing) and their values."""
    codes = np.arange(0x7F)
    return codes, np.array([e4m3_value(c) for c in codes])


def e4m3_encode(v) -> np.ndarray:
    """Nearest e4m3 code of each exact value (ties to the even code, which is
    the even mantissa), saturating to +-448; NaN -> 0x7F. uint8 array."""
    v = np.asarray(v, dtype=np.float64)
    codes, grid = _positive_grid()
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, len(grid) - 1)  # first grid >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    out = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    out = np.where(np.signbit(v) & ~nan, out | 0x80, out)
    return np.where(nan, E4M3_NAN, out).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of an array of codes."""
    return e4m3_table()[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def scale_exponent(amax: float) -> int:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-15, 7]."""
    amax = float(amax)
    if not amax > E4M3_MAX * 2.0 ** SCALE_EXP_MIN:
        return SCALE_EXP_MIN
    e = SCALE_EXP_MIN
    while e < SCALE_EXP_MAX and amax > E4M3_MAX * 2.0 ** e:
        e += 1
    return e


def f16_bits(v) -> np.ndarray:
    """IEEE half bits (uint16) of exact values, rounded to nearest even; values
    beyond the half range become +-inf, as IEEE rounding defines."""
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def f16_value(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def quantize_rows(rows, kv_lora_rank: int):
    """Cache rows (exact values, [n, d_c + d_r]) -> (codes uint8 [n, d_c],
    rope f16 bits uint16 [n, d_r], scale float64 [n] = 2^e)."""
    rows = np.asarray(rows, dtype=np.float64)
    c, pe = rows[:, :kv_lora_rank], rows[:, kv_lora_rank:]
    exps = np.array([scale_exponent(np.max(np.abs(r))) if r.size else SCALE_EXP_MIN for r in c], dtype=np.int64)
    scale = np.ldexp(1.0, exps)
    codes = e4m3_encode(c / scale[:, None])
    return codes, f16_bits(pe), scale


def dequantize_rows(codes, rope_bits, scale) -> np.ndarray:
    """float64 [n, d_c + d_r]: decode(code) * s_t followed by the f16 RoPE key."""
    c = e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]
    return np.concatenate([c, f16_value(rope_bits)], axis=1)


# ----------------------------------------------------------- block layout --
def row_bytes(dims) -> int:
    return dims.kv_lora_rank + 2 * dims.rope_dim


def block_bytes(dims) -> int:
    return dims.block_size * (row_bytes(dims) + 4)


def pack_pool(codes, rope_bits, scale, dims) -> np.ndarray:
    """uint8 [num_blocks, block_bytes] from per-pool-row arrays (row r = block
    r // block_size, token r % block_size)."""
    bs, rb = dims.block_size, row_bytes(dims)
    n = codes.shape[0]
    assert n % bs == 0
    nb = n // bs
    out = np.zeros((nb, block_bytes(dims)), dtype=np.uint8)
    rows = np.concatenate([np.asarray(codes, dtype=np.uint8),
                           np.ascontiguousarray(rope_bits, dtype=np.uint16).view(np.uint8)], axis=1)
    out[:, : bs * rb] = rows.reshape(nb, bs * rb)
    out[:, bs * rb:] = np.asarray(scale, dtype=np.float32).reshape(nb, bs).view(np.uint8)
    return out


def unpack_pool(pool_bytes, dims):
    """Inverse of pack_pool: (codes [rows, d_c], rope bits [rows, d_r], scale float64 [rows])."""
    bs, rb, dc = dims.block_size, row_bytes(dims), dims.kv_lora_rank
    p = np.asarray(pool_bytes, dtype=np.uint8).reshape(-1, block_bytes(dims))
    rows = p[:, : bs * rb].reshape(-1, rb)
    codes = rows[:, :dc]
    rope_bits = np.ascontiguousarray(rows[:, dc:]).view(np.uint16)
    scale = np.ascontiguousarray(p[:, bs * rb:]).view(np.float32).reshape(-1).astype(np.float64)
    return codes, rope_bits, scale


def quantize_pool(pool_values, dims) -> np.ndarray:
    """A cache pool of exact values [num_blocks, block_size, d_c + d_r] in the
    FP8 block layout (uint8 [num_blocks, block_bytes])."""
    rows = np.asarray(pool_values, dtype=np.float64).reshape(-1, dims.kv_lora_rank + dims.rope_dim)
    return pack_pool(*quantize_rows(rows, dims.kv_lora_rank), dims)


def dequantize_pool(pool_bytes, dims) -> np.ndarray:
    """float64 [num_blocks, block_size, d_c + d_r]: the cache the FP8 pool stands for."""
    rows = dequantize_rows(*unpack_pool(pool_bytes, dims))
    return rows.reshape(-1, dims.block_size, dims.kv_lora_rank + dims.rope_dim)
