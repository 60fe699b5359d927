"""GPU checks of the FP8 (e4m3) latent cache through the C ABI.

* mla_cache_to_fp8 against the oracle's quantiser: every byte equal (codes,
  f16 RoPE keys, scales), on rows that reach both ends of the scale range.
* mla_append_kv_fp8 against the oracle's append followed by its quantiser:
  codes within one e4m3 step (the GPU's c comes from an fp32 GEMM, the
  oracle's from fp64, so a rounding decision may differ), and every byte
  outside the written rows and scales untouched.
* mla_decode over the FP8 pool against the fp64 definition on the
  dequantised cache (the oracle's own quantisation of the same bf16 rows,
  checked equal to the GPU's bytes first), with the bf16 tolerance:
  max|err| <= 2e-2 * max|ref| + 1e-3.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_29_b200 import inputs as I
from oracle import fp8_cache as F
from oracle import mla_oracle as O

from _data import build, oracle_append_pool, to_device, tolerance_ok

pytestmark = pytest.mark.gpu


def _lib():
    from mla_latent_kv_29_b200 import lib

    return lib


def _f64(t):
    return t.detach().cpu().double().numpy()


def _v3(name, batch, q_len, lengths, **kw):
    w = I.scaled(I.WORKLOADS["v3_b64_l1k_8k"], batch=batch, q_len=q_len, name=name, **kw)
    return w, torch.tensor(lengths, dtype=torch.int32)


def test_block_bytes():
    L = _lib()
    d = I.WORKLOADS["v3_b64_l1k_8k"].dims
    assert L.fp8_block_bytes(d) == F.block_bytes(d) == 41216
    tiny = I.WORKLOADS["tiny_b1_l128"].dims  # d_r = 16, d_c = 64: supported
    assert L.fp8_block_bytes(tiny) == F.block_bytes(tiny)


def test_cache_to_fp8_is_bit_exact():
    L = _lib()
    d = I.WORKLOADS["v3_b64_l1k_8k"].dims
    g = torch.Generator().manual_seed(4)
    pool = torch.randn(6, 64, 576, generator=g)
    pool[1] *= 2.0 ** -20  # tiny rows: the scale clamps at 2^-15, small codes and subnormals
    pool[2] *= 2.0 ** 14   # huge rows: the scale clamps at 2^7, codes saturate at +-448
    pool[3, :5] = 0.0      # all-zero rows
    pool[4, :, :512] *= torch.logspace(-8, 3, 64, base=2.0)[:, None]  # every exponent in between
    pool = pool.to(torch.bfloat16)
    got = L.cache_to_fp8(d, pool.cuda()).cpu().numpy()
    ref = F.quantize_pool(_f64(pool), d)
    assert got.shape == ref.shape
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:4].tolist()}"


def test_cache_to_fp8_other_dims_is_bit_exact():
    """The conversion is not tied to V3 dims: latent 64, RoPE 16, 128-token blocks."""
    L = _lib()
    d = I.WORKLOADS["tiny_b1_l128"].dims
    g = torch.Generator().manual_seed(6)
    pool = (torch.randn(3, d.block_size, d.row_width, generator=g) * 3.0).to(torch.bfloat16)
    got = L.cache_to_fp8(d, pool.cuda()).cpu().numpy()
    assert np.array_equal(got, F.quantize_pool(_f64(pool), d))


@pytest.mark.parametrize("n_seqs,per_seq,hidden", [(3, 1, 256), (5, 4, 7168), (2, 40, 512)])
def test_append_fp8_matches_oracle_and_touches_only_its_rows(n_seqs, per_seq, hidden):
    L = _lib()
    w = I.scaled(I.WORKLOADS["v3_b16_sq4_l16k_append"], batch=n_seqs, q_len=per_seq, length=300,
                 name=f"append8_{n_seqs}", seed=131 + n_seqs, append_hidden=hidden)
    d = w.dims
    data = build(w, fill=0.0)
    dd = to_device(data)
    nb = data["pool"].shape[0]
    pool8 = torch.full((nb, F.block_bytes(d)), 0xA5, dtype=torch.uint8, device="cuda")  # sentinel bytes
    before = pool8.clone()
    ap = dd["append"]
    L.append_kv(d, ap["x"], ap["w_kva"], ap["seq_ids"], ap["positions"], dd["table"], pool8, fp8=True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    got = pool8.cpu().numpy()
    tab = data["table"].numpy()
    slots = [O.resolve_slot(tab, int(b), int(p), d.block_size)
             for b, p in zip(data["append"]["seq_ids"].tolist(), data["append"]["positions"].tolist())]
    # bytes outside the written rows and their scales are untouched
    touched = np.zeros(got.shape, dtype=bool)
    rb = F.row_bytes(d)
    for r in slots:
        blk, s = divmod(r, d.block_size)
        touched[blk, s * rb:(s + 1) * rb] = True
        touched[blk, d.block_size * rb + 4 * s: d.block_size * rb + 4 * s + 4] = True
    assert np.array_equal(got[~touched], before.cpu().numpy()[~touched])
    # the written rows against the oracle: append in fp64, c rounded to bf16, then quantised
    rows = O.append_rows(data["append"]["x"], data["append"]["w_kva"], data["append"]["positions"].numpy(),
                         d.kv_lora_rank)
    rows[:, :d.kv_lora_rank] = torch.from_numpy(rows[:, :d.kv_lora_rank]).to(torch.bfloat16).double().numpy()
    codes_r, rope_r, scale_r = F.quantize_rows(rows, d.kv_lora_rank)
    codes_g, rope_g, scale_g = F.unpack_pool(got, d)
    codes_g, rope_g, scale_g = codes_g[slots], rope_g[slots], scale_g[slots]
    # the scale is a power of two chosen from the row maximum: equal unless that
    # maximum sits within rounding of a power-of-two boundary
    assert np.all((scale_g == scale_r) | (scale_g == 2 * scale_r) | (2 * scale_g == scale_r))
    assert np.mean(scale_g == scale_r) > 0.9
    deq_g = F.dequantize_rows(codes_g, rope_g, scale_g)
    deq_r = F.dequantize_rows(codes_r, rope_r, scale_r)
    c_g, c_r = deq_g[:, :d.kv_lora_rank], deq_r[:, :d.kv_lora_rank]
    s = np.maximum(scale_g, scale_r)[:, None]
    # one e4m3 step (2^-3 relative, or the subnormal step) plus the bf16 rounding of c
    assert np.all(np.abs(c_g - c_r) <= 2.0 ** -3 * np.abs(c_r) + 2.0 ** -9 * s + 2.0 ** -7 * np.abs(c_r))
    assert np.mean(codes_g == codes_r) > 0.95
    pe_g, pe_r = deq_g[:, d.kv_lora_rank:], rows[:, d.kv_lora_rank:]
    assert np.all(np.abs(pe_g - pe_r) <= 2.0 ** -10 * np.abs(pe_r) + 2e-3)  # f16 of an fp32 RoPE


def _fp8_pools(w, data):
    """(GPU bytes from mla_cache_to_fp8, the oracle's dequantised pool) of the
    workload's bf16 pool; the finite rows' bytes must agree exactly."""
    L = _lib()
    d = w.dims
    pool = data["pool"]
    got = L.cache_to_fp8(d, pool.cuda())
    ref = F.quantize_pool(_f64(pool), d)
    g = got.cpu().numpy()
    finite = np.isfinite(_f64(pool)).all(axis=-1)  # per row
    rb = F.row_bytes(d)
    for blk in range(g.shape[0]):
        for s in np.nonzero(finite[blk])[0]:
            assert np.array_equal(g[blk, s * rb:(s + 1) * rb], ref[blk, s * rb:(s + 1) * rb])
            o = d.block_size * rb + 4 * s
            assert np.array_equal(g[blk, o:o + 4], ref[blk, o:o + 4])
    return got, F.dequantize_pool(ref, d)


def _check(got, ref, ids=None):
    if ids is not None:
        got, ref = got[ids], ref[ids]
    assert np.all(np.isfinite(got))
    ok, err, bound = tolerance_ok(got, ref)
    assert ok, f"max|err| {err:.3e} > {bound:.3e}"


def _decode8(w, dd, pool8, workers=0):
    L = _lib()
    out = L.decode(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], pool8, dd["table"], dd["lengths"],
                   int(dd["lengths"].max()), dd["w_uk"], dd["w_uv"], num_workers=workers, cache_fp8=True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    return out.float().cpu().numpy()


@pytest.mark.parametrize("case", [
    ("ragged_sq1", 3, 1, [1, 65, 300]),
    ("ragged_sq4", 2, 4, [4, 130]),
    ("tiles_exact", 2, 1, [128, 256]),
    ("one_page_tail", 4, 2, [63, 64, 65, 129]),
    ("prefill_chunk", 2, 128, [128, 700]),
])
@pytest.mark.parametrize("workers", [0, 1, 5])
def test_fp8_decode_small_cases(case, workers):
    name, B, sq, lens = case
    w, lengths = _v3(name + "_f8", B, sq, lens)
    data = build(w, lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    got = _decode8(w, to_device(data), pool8, workers)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], w.dims, w.softmax_scale)
    _check(got, ref)


def test_fp8_decode_ignores_nan_rows_outside_the_context():
    w, lengths = _v3("nan_fill_f8", 3, 2, [70, 5, 200], spare_blocks=3)
    data = build(w, fill=float("nan"), lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    got = _decode8(w, to_device(data), pool8, workers=7)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], w.dims, w.softmax_scale)
    _check(got, ref)


def test_fp8_decode_after_fp8_append():
    """The step on the FP8 cache: old tokens converted, the new ones appended
    by mla_append_kv_fp8, then the decode; against the oracle's append,
    quantised, and the definition."""
    L = _lib()
    w = I.scaled(I.WORKLOADS["v3_b16_sq4_l16k_append"], batch=3, q_len=4, length=500, name="append_decode_f8",
                 seed=171)
    d = w.dims
    data = build(w, fill=0.0)
    dd = to_device(data)
    pool8 = L.cache_to_fp8(d, dd["pool"])
    ap = dd["append"]
    L.append_kv(d, ap["x"], ap["w_kva"], ap["seq_ids"], ap["positions"], dd["table"], pool8, fp8=True)
    got = _decode8(w, dd, pool8)
    ref_pool = oracle_append_pool(w, data)  # appended rows rounded to bf16, as the FP8 append does before quantising
    deq = F.dequantize_pool(F.quantize_pool(_f64(ref_pool), d), d)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], d, w.softmax_scale)
    _check(got, ref)


def test_fp8_decode_needs_the_tensor_core_kernel():
    L = _lib()
    w, lengths = _v3("f8_generic", 1, 1, [100])
    data = build(w, lengths=lengths)
    dd = to_device(data)
    pool8 = L.cache_to_fp8(w.dims, dd["pool"])
    with pytest.raises(L.MLAError) as e:
        L.decode(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], pool8, dd["table"], dd["lengths"], 100,
                 dd["w_uk"], dd["w_uv"], kernel=2, cache_fp8=True)
    assert e.value.status == -2


def test_fp8_full_size_sampled():
    """The batch-64 workload over its FP8 cache: three sampled sequences, all heads."""
    L = _lib()
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    d = w.dims
    data = build(w)
    dd = to_device(data)
    pool8 = L.cache_to_fp8(d, dd["pool"])
    got = _decode8(w, dd, pool8)
    g = torch.Generator().manual_seed(w.seed + 78)
    ids = sorted(torch.randperm(w.batch, generator=g)[:3].tolist())
    # the oracle quantises only the sampled sequences' rows
    tab = data["table"].numpy()
    flat = data["pool"].view(-1, d.row_width)
    deq = np.zeros((data["pool"].shape[0] * d.block_size, d.row_width))
    g8 = pool8.cpu().numpy()
    codes_g, rope_g, scale_g = F.unpack_pool(g8, d)
    for b in ids:
        rows = np.array([O.resolve_slot(tab, b, t, d.block_size) for t in range(int(data["lengths"][b]))])
        codes, rope, scale = F.quantize_rows(_f64(flat[torch.from_numpy(rows)]), d.kv_lora_rank)
        assert np.array_equal(codes, codes_g[rows]) and np.array_equal(rope, rope_g[rows])
        assert np.array_equal(scale, scale_g[rows])
        deq[rows] = F.dequantize_rows(codes, rope, scale)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq.reshape(-1, d.block_size, d.row_width), tab,
                         data["lengths"], data["w_uk"], data["w_uv"], d, w.softmax_scale, batch_ids=ids)
    _check(got, ref, ids=ids)


def test_fp8_bounded_wait_expiry_reports_timeout_and_context_survives():
    """The FP8 kernel's waits give up too: with its load warps starved and a 1 ms
    limit, every role (expansion warps included) drains and the call reports
    MLA_ERR_DEVICE_TIMEOUT; an ordinary FP8 decode afterwards still matches."""
    L = _lib()
    w, lengths = _v3("f8_wait_expiry", 1, 1, [100])
    data = build(w, lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    dd = to_device(data)
    L.device_error()  # clear
    L.decode(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], pool8, dd["table"], dd["lengths"], 100,
             dd["w_uk"], dd["w_uv"], kernel=1, debug_wait_limit_us=1000, debug_starve=True, cache_fp8=True)
    assert L.device_error() == -6
    assert L.device_error() == 0
    got = _decode8(w, dd, pool8)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], w.dims, w.softmax_scale)
    _check(got, ref)


def test_fp8_decode_latent_output():
    """With output_latent the FP8 decode returns o_lat: the oracle's latent decode
    on the dequantised cache."""
    L = _lib()
    w, lengths = _v3("f8_latent", 3, 2, [300, 77, 129])
    data = build(w, lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    dd = to_device(data)
    o_lat = L.decode(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], pool8, dd["table"], dd["lengths"], 300,
                     dd["w_uk"], dd["w_uv"], output_latent=True, cache_fp8=True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.decode_latent_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"],
                                data["w_uk"], w.dims, w.softmax_scale)
    _check(o_lat.float().cpu().numpy(), ref)


def test_fp8_decode_without_a_workspace():
    """mla_decode_no_alloc reads the FP8 cache too (its scratch is the library's
    own buffer); against the oracle on the dequantised cache."""
    L = _lib()
    w, lengths = _v3("f8_no_alloc", 4, 2, [63, 64, 65, 129])
    data = build(w, lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    dd = to_device(data)
    got = L.decode_no_alloc(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], pool8, dd["table"], dd["lengths"],
                            129, dd["w_uk"], dd["w_uv"], cache_fp8=True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], w.dims, w.softmax_scale)
    _check(got.float().cpu().numpy(), ref)


def test_fp8_decode_pages_of_128_tokens():
    """The FP8 maps address (slot, block): 128-token pages put a tile's halves
    at slots 0 and 64 of one block."""
    import dataclasses

    w, lengths = _v3("f8_pages128", 3, 2, [70, 260, 385])
    w = dataclasses.replace(w, dims=dataclasses.replace(w.dims, block_size=128))
    data = build(w, lengths=lengths)
    pool8, deq = _fp8_pools(w, data)
    got = _decode8(w, to_device(data), pool8, workers=3)
    ref = O.decode_paged(data["q_nope"], data["q_pe"], deq, data["table"].numpy(), data["lengths"], data["w_uk"],
                         data["w_uv"], w.dims, w.softmax_scale)
    _check(got, ref)
