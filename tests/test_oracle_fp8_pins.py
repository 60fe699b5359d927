"""Pins for the FP8 cache oracle (``oracle.fp8_cache``).

The e4m3 decoder and encoder are tied to the format's defining values and
to PyTorch's float8_e4m3fn conversion (a library routine outside this
repository); the scale rule to its closed form; the block layout to a
round trip; and attention over the FP8 cache to the bf16 definition on a
cache whose values the format holds exactly.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp8_cache as F
from oracle import mla_oracle as O
from mla_latent_kv_29_b200 import inputs as I


def test_e4m3_defining_values():
    v = F.e4m3_value
    assert v(0x00) == 0.0 and v(0x80) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert v(0x38) == 1.0  # exponent field 7 = bias, mantissa 0
    assert v(0x01) == 2.0 ** -9  # smallest subnormal
    assert v(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert v(0x08) == 2.0 ** -6  # smallest normal
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0  # largest finite
    assert v(0x3C) == 1.5 and v(0xC0) == -2.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    _, grid = F._positive_grid()
    assert len(grid) == 127 and np.all(np.diff(grid) > 0)  # 0x00..0x7E strictly increasing


def test_e4m3_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = F.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(mine[~nan]))


def test_e4m3_encode_matches_torch_rounding():
    rng = np.random.default_rng(5)
    _, grid = F._positive_grid()
    mids = (grid[1:] + grid[:-1]) / 2  # exact ties: the even code must win
    vals = np.concatenate([grid, mids, -mids, rng.uniform(-448, 448, 20000),
                           rng.normal(0, 1, 20000), rng.normal(0, 2.0 ** -7, 5000), [0.0, -0.0, 464.0, -464.0]])
    vals = vals.astype(np.float32).astype(np.float64)  # exactly representable in fp32 for the torch cast
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(vals), ref)


def test_e4m3_encode_saturates_and_ties_to_even():
    assert F.e4m3_encode([500.0, 1e9, -1e9, 449.0])[:].tolist() == [0x7E, 0x7E, 0xFE, 0x7E]
    assert F.e4m3_encode([1.0625])[0] == 0x38  # halfway 1 and 1.125: even mantissa 0
    assert F.e4m3_encode([1.1875])[0] == 0x3A  # halfway 1.125 and 1.25: even mantissa 2
    assert F.e4m3_encode([2.0 ** -10])[0] == 0x00  # half the smallest subnormal -> 0 (even)
    assert F.e4m3_encode([3 * 2.0 ** -10])[0] == 0x02  # halfway codes 1 and 2 -> 2
    assert F.e4m3_encode([math.nan])[0] == 0x7F  # S.1111.111, the code torch's cast gives too
    assert torch.tensor([math.nan]).to(torch.float8_e4m3fn).view(torch.uint8).item() == 0x7F


def test_scale_exponent_closed_form():
    assert F.scale_exponent(448.0) == 0
    assert F.scale_exponent(448.0 * (1 + 2 ** -20)) == 1
    assert F.scale_exponent(224.0) == -1
    assert F.scale_exponent(224.5) == 0
    assert F.scale_exponent(0.0) == -15
    assert F.scale_exponent(1e-30) == -15
    assert F.scale_exponent(1e9) == 7
    rng = np.random.default_rng(3)
    for a in rng.lognormal(0, 3, 2000):
        e = F.scale_exponent(a)
        if F.SCALE_EXP_MIN < e < F.SCALE_EXP_MAX:
            assert 448.0 * 2.0 ** (e - 1) < a <= 448.0 * 2.0 ** e
            assert e == math.ceil(math.log2(a / 448.0)) or a == 448.0 * 2.0 ** e


def test_quantize_error_bound_and_grid_round_trip():
    rng = np.random.default_rng(11)
    rows = np.concatenate([rng.normal(0, 1, (300, 512)), rng.normal(0, 1, (300, 64))], axis=1)
    rows = torch.from_numpy(rows).to(torch.bfloat16).double().numpy()
    codes, rope_bits, scale = F.quantize_rows(rows, 512)
    back = F.dequantize_rows(codes, rope_bits, scale)
    c, cb = rows[:, :512], back[:, :512]
    s = scale[:, None]
    normal = np.abs(c) >= 2.0 ** -6 * s
    assert np.all(np.abs(cb - c)[normal] <= 2.0 ** -4 * np.abs(c)[normal])  # half an ulp of 3 mantissa bits
    assert np.all(np.abs(cb - c)[~normal] <= 2.0 ** -10 * np.broadcast_to(s, c.shape)[~normal])
    assert np.all(np.max(np.abs(cb), axis=1) <= 448.0 * scale)
    assert np.all(np.max(np.abs(c), axis=1) > 224.0 * scale)  # the scale is the tightest power of two
    assert np.array_equal(back[:, 512:], rows[:, 512:].astype(np.float16).astype(np.float64))
    # values already on the scaled grid come back exactly
    again = F.dequantize_rows(*F.quantize_rows(back, 512))
    assert np.array_equal(again, back)


def test_pool_layout_round_trip_and_size():
    d = I.WORKLOADS["v3_b64_l1k_8k"].dims
    assert F.row_bytes(d) == 640 and F.block_bytes(d) == 41216
    rng = np.random.default_rng(2)
    pool = torch.from_numpy(rng.normal(0, 1, (3, 64, 576))).to(torch.bfloat16).double().numpy()
    packed = F.quantize_pool(pool, d)
    assert packed.shape == (3, 41216) and packed.dtype == np.uint8
    codes, rope_bits, scale = F.unpack_pool(packed, d)
    assert np.array_equal(F.pack_pool(codes, rope_bits, scale, d), packed)
    # the first row's codes and its scale sit where the layout says
    row0 = F.quantize_rows(pool[0, :1].reshape(1, -1), 512)
    assert np.array_equal(packed[0, :512], row0[0][0])
    assert np.frombuffer(packed[0, 64 * 640:64 * 640 + 4].tobytes(), dtype=np.float32)[0] == row0[2][0]
    assert np.frombuffer(packed[1, 640 + 512:640 + 514].tobytes(), dtype=np.uint16)[0] == \
        F.f16_bits(pool[1, 1, 512:513])[0]


def test_fp8_attention_is_the_definition_on_an_exact_cache():
    """On a cache whose latent values are e4m3 grid points times 2^-4 (row
    maxima in (14, 28]) and whose RoPE keys are both bf16 and f16 values, quantising loses
    nothing, so attention over the FP8 pool equals the bf16 definition."""
    w = I.scaled(I.WORKLOADS["v3_b64_l1k_8k"], batch=2, q_len=2, name="fp8_exact")
    d = w.dims
    dims = I.Dims(num_heads=4, kv_lora_rank=d.kv_lora_rank, rope_dim=d.rope_dim, qk_nope_dim=d.qk_nope_dim,
                  v_head_dim=d.v_head_dim, block_size=d.block_size)
    rng = np.random.default_rng(9)
    nb = 4
    codes = rng.integers(0, 0x7F, (nb * 64, 512)).astype(np.uint8)
    codes[:, 0] = 0x7E - rng.integers(0, 8, nb * 64)  # a code in (224, 448]: the row's scale is 2^-4
    codes |= (rng.integers(0, 2, codes.shape) << 7).astype(np.uint8)
    c = F.e4m3_decode(codes) * 2.0 ** -4
    pe = torch.from_numpy(rng.normal(0, 1, (nb * 64, 64))).to(torch.bfloat16).double().numpy()
    pe[np.abs(pe) < 2.0 ** -14] = 0.0  # bf16 values in the f16 normal range are exact halves
    pool = np.concatenate([c, pe], axis=1).reshape(nb, 64, 576)
    assert np.array_equal(torch.from_numpy(pool).to(torch.bfloat16).double().numpy(), pool)  # bf16-exact
    packed = F.quantize_pool(pool, dims)
    assert np.array_equal(F.dequantize_pool(packed, dims), pool)
    table = np.array([[2, 0], [3, 1]], dtype=np.int32)
    lengths = [100, 77]
    q_nope = rng.normal(0, 1, (2, 2, 4, 128))
    q_pe = rng.normal(0, 1, (2, 2, 4, 64))
    w_uk = rng.normal(0, 512 ** -0.5, (4, 128, 512))
    w_uv = rng.normal(0, 512 ** -0.5, (4, 128, 512))
    a = O.decode_paged(q_nope, q_pe, F.dequantize_pool(packed, dims), table, lengths, w_uk, w_uv, dims,
                       w.softmax_scale)
    b = O.decode_paged(q_nope, q_pe, pool, table, lengths, w_uk, w_uv, dims, w.softmax_scale)
    assert np.array_equal(a, b)
    # a cache the format does not hold exactly moves the result (the quantiser is not the identity)
    pool2 = pool.copy()
    pool2[..., 1] += 2.0 ** -12
    c2 = F.dequantize_pool(F.quantize_pool(pool2, dims), dims)
    assert not np.array_equal(c2, pool2)
