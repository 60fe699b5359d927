"""GPU parity of the non-decode entry points through the C ABI: the split-KV
combine, the page resolver (bit-exact) and the fused cache append."""
import math

import numpy as np
import pytest
import torch

from mla_latent_kv_29_b200 import inputs as I
from oracle import mla_oracle as O

from _data import build, oracle_append_pool, to_device, tolerance_ok

pytestmark = pytest.mark.gpu


def _lib():
    from mla_latent_kv_29_b200 import lib

    return lib


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("dims", [I.V3, I.TINY])
def test_combine_matches_oracle_merge(dims):
    L = _lib()
    g = torch.Generator().manual_seed(4242)
    counts = [1, 3, 0, 7, 2, 64, 65, 1]  # 0: a group with no parts; 65: more than one merge chunk
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    n, H, dc = int(offs[-1]), dims.num_heads, dims.kv_lora_rank
    o = torch.randn(n, H, dc, generator=g)
    lse = torch.randn(n, H, generator=g) * 4
    lse[offs[1]:offs[2]][1] = -math.inf          # an empty split
    lse[offs[4]:offs[5]] = -math.inf             # a group whose parts are all empty
    dev = "cuda"
    lse_out = torch.empty(len(counts), H, device=dev)
    got = L.combine(dims, o.to(dev), lse.to(dev), torch.from_numpy(offs).to(dev), lse_out=lse_out)
    torch.cuda.synchronize()
    got, lse_got = got.cpu().numpy(), lse_out.cpu().numpy()
    for gi in range(len(counts)):
        a, b = offs[gi], offs[gi + 1]
        if a == b:
            np.testing.assert_array_equal(got[gi], 0.0)
            assert np.all(lse_got[gi] == -np.inf)
            continue
        ref, ref_lse = O.merge_partials(o[a:b].numpy(), lse[a:b].numpy())
        ok, err, bound = tolerance_ok(got[gi], ref)
        assert ok, (gi, err, bound)
        finite = np.isfinite(ref_lse)
        np.testing.assert_array_equal(np.isfinite(lse_got[gi]), finite)
        np.testing.assert_allclose(lse_got[gi][finite], ref_lse[finite], rtol=1e-5, atol=1e-5)


# ---------------------------------------------------------------- resolver
def test_resolve_slots_bit_exact():
    L = _lib()
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    lengths = I.context_lengths(w)
    table, nblk = I.block_table(w, lengths)
    g = torch.Generator().manual_seed(9)
    n = 20000
    seq = torch.randint(0, w.batch, (n,), generator=g, dtype=torch.int32)
    pos = (torch.rand(n, generator=g) * lengths[seq.long()].float()).to(torch.int32)
    # out-of-range probes: sequence, negative position, position past the table row
    seq = torch.cat([seq, torch.tensor([-1, 64, 0, 0], dtype=torch.int32)])
    pos = torch.cat([pos, torch.tensor([0, 0, -3, table.shape[1] * 64], dtype=torch.int32)])
    rows = L.resolve_slots(w.dims, table.cuda(), nblk, seq.cuda(), pos.cuda()).cpu()
    tab = table.numpy()
    ref = [O.resolve_slot(tab, int(b), int(t), 64) for b, t in zip(seq[:n].tolist(), pos[:n].tolist())]
    assert rows[:n].tolist() == ref
    assert rows[n:].tolist() == [-1, -1, -1, -1]


# ------------------------------------------------------------------ append
def _append_case(n_seqs, per_seq, hidden, seed):
    w = I.scaled(I.WORKLOADS["v3_b16_sq4_l16k_append"], batch=n_seqs, q_len=per_seq, length=300,
                 name=f"append_{seed}", seed=seed, append_hidden=hidden)
    return w


@pytest.mark.parametrize("n_seqs,per_seq,hidden", [(3, 1, 256), (5, 4, 7168), (16, 4, 7168), (2, 40, 512),
                                                   (3, 50, 320), (10, 110, 512)])
def test_append_matches_oracle_and_touches_only_its_rows(n_seqs, per_seq, hidden):
    L = _lib()
    w = _append_case(n_seqs, per_seq, hidden, 31 + n_seqs)
    data = build(w, fill=float("nan"))
    ref_pool = oracle_append_pool(w, data)
    dd = to_device(data)
    before = dd["pool"].clone()
    ap = dd["append"]
    L.append_kv(w.dims, ap["x"], ap["w_kva"], ap["seq_ids"], ap["positions"], dd["table"], dd["pool"])
    torch.cuda.synchronize()
    assert L.device_error() == 0
    after = dd["pool"].cpu()
    d = w.dims
    flat_a, flat_b = after.view(-1, d.row_width), before.cpu().view(-1, d.row_width)
    tab = data["table"].numpy()
    slots = [O.resolve_slot(tab, int(b), int(p), d.block_size)
             for b, p in zip(data["append"]["seq_ids"].tolist(), data["append"]["positions"].tolist())]
    mask = torch.ones(flat_a.shape[0], dtype=torch.bool)
    mask[slots] = False
    # every other row is untouched, bit for bit (NaN sentinels included)
    assert torch.equal(flat_a[mask].view(torch.int16), flat_b[mask].view(torch.int16))
    # the written rows match the oracle's fp64 rows
    ref_rows = O.append_rows(data["append"]["x"], data["append"]["w_kva"], data["append"]["positions"].numpy(),
                             d.kv_lora_rank)
    got = flat_a[slots].float().numpy()
    ok, err, bound = tolerance_ok(got, ref_rows)
    assert ok, (err, bound)
    # elementwise: one bf16 rounding plus fp32 accumulation error
    assert np.all(np.abs(got - ref_rows) <= 2.0 ** -8 * np.abs(ref_rows) + 2e-3)
    # and the oracle's own bf16 storage of those rows differs by at most one bf16 step
    ref_bf16 = ref_pool.view(-1, d.row_width)[slots].float().numpy()
    assert np.all(np.abs(got - ref_bf16) <= 2.0 ** -7 * np.abs(ref_bf16) + 1e-3)


def test_append_bad_slot_is_skipped_and_reported():
    L = _lib()
    w = _append_case(2, 2, 128, 77)
    data = build(w, fill=0.0)
    data["append"]["seq_ids"][1] = 5  # no such sequence
    dd = to_device(data)
    before = dd["pool"].clone()
    ap = dd["append"]
    L.device_error()
    L.append_kv(w.dims, ap["x"], ap["w_kva"], ap["seq_ids"], ap["positions"], dd["table"], dd["pool"])
    assert L.device_error() == -5
    changed = (dd["pool"] != before).any(-1).view(-1).sum().item()
    assert changed == 3  # the three valid tokens were written


def test_append_tiny_dims_uses_the_cuda_core_path():
    """d_c + d_r = 80 is not a multiple of the tensor-core tile: exercises the CUDA-core GEMM."""
    L = _lib()
    w = I.scaled(I.WORKLOADS["tiny_b1_l128"], batch=2, q_len=3, length=128, name="append_tiny", seed=91,
                 append_hidden=96, append_w_std=96 ** -0.5)
    data = build(w, fill=float("nan"))
    dd = to_device(data)
    ap = dd["append"]
    L.append_kv(w.dims, ap["x"], ap["w_kva"], ap["seq_ids"], ap["positions"], dd["table"], dd["pool"])
    torch.cuda.synchronize()
    assert L.device_error() == 0
    d = w.dims
    tab = data["table"].numpy()
    slots = [O.resolve_slot(tab, int(b), int(p), d.block_size)
             for b, p in zip(data["append"]["seq_ids"].tolist(), data["append"]["positions"].tolist())]
    got = dd["pool"].view(-1, d.row_width)[torch.tensor(slots, device="cuda")].float().cpu().numpy()
    ref = O.append_rows(data["append"]["x"], data["append"]["w_kva"], data["append"]["positions"].numpy(),
                        d.kv_lora_rank)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-3)


# -------------------------------------------------------- query projection
@pytest.mark.parametrize("case", [
    ("small", I.Dims(num_heads=4, kv_lora_rank=64, rope_dim=32, qk_nope_dim=32, v_head_dim=32, block_size=64),
     5, 256, 128, True),
    # RoPE width 64 and d_n a multiple of 64: the second product writes the heads itself
    ("small_heads_in_gemm", I.Dims(num_heads=4, kv_lora_rank=64, rope_dim=64, qk_nope_dim=64, v_head_dim=32,
                                   block_size=64), 5, 256, 128, True),
    ("v3", I.WORKLOADS["v3_b64_l1k_8k"].dims, 64, 7168, 1536, True),
    ("v3_ragged_no_gamma", I.WORKLOADS["v3_b64_l1k_8k"].dims, 130, 7168, 1536, False),
])
def test_q_proj_matches_oracle(case):
    """mla_q_proj against the oracle's fp64 query projection, q_nope and q_pe
    each within the decode tolerance and elementwise within a few bf16 steps."""
    L = _lib()
    _, d, T, hidden, rank, with_gamma = case
    inp = I.q_proj_inputs(d, T, hidden, rank, seed=41 + T, gamma=with_gamma)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    qn, qp = L.q_proj(d, dev["x"], dev["w_qa"], dev["w_qb"], dev["positions"], q_gamma=dev["gamma"])
    torch.cuda.synchronize()
    assert L.device_error() == 0
    ref_n, ref_p = O.query_projection(inp["x"], inp["w_qa"], inp["w_qb"], inp["positions"].numpy(), d.num_heads,
                                      d.qk_nope_dim, d.rope_dim, gamma=inp["gamma"])
    for got, ref in ((qn, ref_n), (qp, ref_p)):
        got = got.float().cpu().numpy()
        assert got.shape == ref.shape
        ok, err, bound = tolerance_ok(got, ref)
        assert ok, (err, bound)
        # c_q is rounded to bf16 before the second product and the result once more
        scale = np.abs(ref).max()
        assert np.all(np.abs(got - ref) <= 2.0 ** -6 * np.abs(ref) + 2.0 ** -8 * scale)


# ------------------------------------------------------- output projection
def _check(got, ref):
    got = got.float().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert np.all(np.isfinite(got))
    ok, err, bound = tolerance_ok(got, ref)
    assert ok, f"max|err| {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("T,K,N", [(1, 256, 128), (64, 2048, 576), (130, 1024, 320), (64, 16384, 256)])
def test_o_proj_matches_oracle(T, K, N):
    """mla_o_proj y = bf16(x W) against the oracle's output projection (x read as
    heads of 64 values), over row tiles, ragged rows and several K splits."""
    L = _lib()
    g = torch.Generator().manual_seed(T * 7 + K + N)
    x = I.bf16(torch.randn(T, K, generator=g))
    w = I.bf16(torch.randn(K, N, generator=g) / math.sqrt(K))
    y = L.o_proj(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert L.device_error() == 0
    _check(y, O.output_projection(x.view(T, K // 64, 64), w))


def test_output_projection_after_decode_unfused_and_absorbed():
    """The decode output through W_O, and the full absorption: the decode's o_lat
    (output_latent) through W_UV^T W_O; both against the oracle's explicit
    decode followed by the output projection, and o_lat against the oracle's
    latent decode."""
    L = _lib()
    w = I.scaled(I.WORKLOADS["v3_b64_l1k_8k"], batch=3, q_len=2, name="o_proj_chain")
    data = build(w, lengths=torch.tensor([300, 77, 129], dtype=torch.int32))
    dd = to_device(data)
    d = w.dims
    hidden = 256
    g = torch.Generator().manual_seed(31)
    w_o = I.bf16(torch.randn(d.num_heads * d.v_head_dim, hidden, generator=g) / math.sqrt(d.num_heads * d.v_head_dim))
    args = (d, w.softmax_scale, dd["q_nope"], dd["q_pe"], dd["pool"], dd["table"], dd["lengths"], 300,
            dd["w_uk"], dd["w_uv"])
    explicit = O.decode_paged(data["q_nope"], data["q_pe"], data["pool"], data["table"].numpy(), data["lengths"],
                              data["w_uk"], data["w_uv"], d, w.softmax_scale)
    ref_y = O.output_projection(explicit, w_o).reshape(-1, hidden)
    out = L.decode(*args)
    y = L.o_proj(out, w_o.cuda())
    torch.cuda.synchronize()
    assert L.device_error() == 0
    _check(y, ref_y)
    o_lat = L.decode(*args, output_latent=True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert tuple(o_lat.shape) == (3, 2, d.num_heads, d.kv_lora_rank)
    _check(o_lat, O.decode_latent_paged(data["q_nope"], data["q_pe"], data["pool"], data["table"].numpy(),
                                        data["lengths"], data["w_uk"], d, w.softmax_scale))
    w_f = torch.from_numpy(O.absorbed_output_weight(data["w_uv"], w_o)).to(torch.bfloat16)
    y_f = L.o_proj(o_lat, w_f.cuda())
    torch.cuda.synchronize()
    assert L.device_error() == 0
    _check(y_f, ref_y)


def test_output_latent_needs_the_tensor_core_merge():
    L = _lib()
    w = I.WORKLOADS["tiny_b1_l128"]
    dd = to_device(build(w))
    with pytest.raises(L.MLAError) as e:
        L.decode(w.dims, w.softmax_scale, dd["q_nope"], dd["q_pe"], dd["pool"], dd["table"], dd["lengths"], 128,
                 dd["w_uk"], dd["w_uv"], output_latent=True)
    assert e.value.status == -2
