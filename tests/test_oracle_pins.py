"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties one oracle function to a brute-force loop, a closed form, a
mathematical identity or a textbook routine, chosen so that a plausible slip
(a dropped score term, a transposed weight, a wrong RoPE pairing or sign, an
off-by-one in the causal window, a wrong combine weight) fails at least one.
"""
import math

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from mla_latent_kv_29_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _rng(seed):
    return np.random.default_rng(seed)


def _small_dims(H=3, dc=6, dr=4, dn=5, dv=3, bs=4):
    return I.Dims(num_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope_dim=dn, v_head_dim=dv,
                  block_size=bs)


# ------------------------------------------------------------------------
# 1. brute force: pure-Python loops over every index
# ------------------------------------------------------------------------
def _brute_decode(q_nope, q_pe, c, kpe, w_uk, w_uv, scale):
    """Explicit MLA decode with nothing but Python scalar loops."""
    sq, H, dn = len(q_nope), len(q_nope[0]), len(q_nope[0][0])
    L, dc, dr = len(c), len(c[0]), len(kpe[0])
    dv = len(w_uv[0])
    out = [[[0.0] * dv for _ in range(H)] for _ in range(sq)]
    for s in range(sq):
        last = L - sq + s  # last visible token index
        for h in range(H):
            scores = []
            for t in range(last + 1):
                acc = 0.0
                for i in range(dn):  # k_nope[t][i] = sum_j W_UK[h][i][j] c[t][j]
                    k = 0.0
                    for j in range(dc):
                        k += w_uk[h][i][j] * c[t][j]
                    acc += q_nope[s][h][i] * k
                for r in range(dr):
                    acc += q_pe[s][h][r] * kpe[t][r]
                scores.append(acc * scale)
            mx = max(scores)
            ex = [math.exp(z - mx) for z in scores]
            tot = sum(ex)
            for i in range(dv):
                val = 0.0
                for t in range(last + 1):
                    v = 0.0
                    for j in range(dc):
                        v += w_uv[h][i][j] * c[t][j]
                    val += ex[t] / tot * v
                out[s][h][i] = val
    return out


def test_bruteforce_decode_paged():
    d = _small_dims()
    rng = _rng(1)
    B, sq = 2, 2
    lengths = [7, 3]
    nblk = [2, 1]
    table = np.array([[3, 0], [1, -1]], dtype=np.int32)
    pool = rng.standard_normal((4, d.block_size, d.row_width))
    q_nope = rng.standard_normal((B, sq, d.num_heads, d.qk_nope_dim))
    q_pe = rng.standard_normal((B, sq, d.num_heads, d.rope_dim))
    w_uk = rng.standard_normal((d.num_heads, d.qk_nope_dim, d.kv_lora_rank)) * 0.4
    w_uv = rng.standard_normal((d.num_heads, d.v_head_dim, d.kv_lora_rank)) * 0.4
    scale = 1.0 / math.sqrt(d.qk_nope_dim + d.rope_dim)
    got = O.decode_paged(q_nope, q_pe, pool, table, lengths, w_uk, w_uv, d, scale)
    for b in range(B):
        rows = []
        for t in range(lengths[b]):  # page walk written out independently
            blk = table[b][t // d.block_size]
            rows.append(pool[blk, t % d.block_size])
        c = [list(r[: d.kv_lora_rank]) for r in rows]
        kpe = [list(r[d.kv_lora_rank:]) for r in rows]
        ref = np.array(_brute_decode(q_nope[b].tolist(), q_pe[b].tolist(), c, kpe,
                                     w_uk.tolist(), w_uv.tolist(), scale))
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-13)
    assert nblk == [2, 1]


def test_bruteforce_append():
    rng = _rng(2)
    T, hid, dc, dr = 3, 5, 4, 4
    x = rng.standard_normal((T, hid))
    w = rng.standard_normal((hid, dc + dr))
    pos = [0, 1, 7]
    got = O.append_rows(x, w, pos, dc, eps=1e-6)
    for t in range(T):
        kv = [sum(x[t][k] * w[k][n] for k in range(hid)) for n in range(dc + dr)]
        ms = sum(v * v for v in kv[:dc]) / dc
        c = [v / math.sqrt(ms + 1e-6) for v in kv[:dc]]
        pe = kv[dc:]
        half = dr // 2
        out = [0.0] * dr
        for i in range(half):
            th = pos[t] * 10000.0 ** (-2.0 * i / dr)
            out[i] = pe[i] * math.cos(th) - pe[i + half] * math.sin(th)
            out[i + half] = pe[i + half] * math.cos(th) + pe[i] * math.sin(th)
        np.testing.assert_allclose(got[t], c + out, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------
# 2. closed-form absorption identity (explicit == absorbed)
# ------------------------------------------------------------------------
@pytest.mark.parametrize("H,dc,dr,dn,dv,L,sq", [(4, 32, 8, 16, 16, 50, 3), (8, 128, 32, 64, 64, 16, 1)])
def test_absorption_identity(H, dc, dr, dn, dv, L, sq):
    rng = _rng(3)
    q_nope = rng.standard_normal((sq, H, dn))
    q_pe = rng.standard_normal((sq, H, dr))
    c = rng.standard_normal((L, dc))
    kpe = rng.standard_normal((L, dr))
    w_uk = rng.standard_normal((H, dn, dc)) / math.sqrt(dc)
    w_uv = rng.standard_normal((H, dv, dc)) / math.sqrt(dc)
    scale = 1.0 / math.sqrt(dn + dr)
    explicit = O.decode_sequence(q_nope, q_pe, c, kpe, w_uk, w_uv, scale)
    q_lat = O.absorb_query(q_nope, w_uk)  # [sq, H, dc]
    o_lat = np.zeros((sq, H, dc))
    for s in range(sq):
        n = L - sq + s + 1
        for h in range(H):
            o_lat[s, h], _ = O.latent_partial(q_lat[s, h], q_pe[s, h], c[:n], kpe[:n], scale)
    absorbed = O.up_project(o_lat, w_uv)
    np.testing.assert_allclose(absorbed, explicit, rtol=1e-10, atol=1e-12)


def test_absorption_detects_transposed_weight():
    """The identity is sharp: using W_UK^T in place of W_UK breaks it."""
    rng = _rng(4)
    H, d = 2, 8
    q_nope = rng.standard_normal((1, H, d))
    q_pe = rng.standard_normal((1, H, 4))
    c = rng.standard_normal((9, d))
    kpe = rng.standard_normal((9, 4))
    w = rng.standard_normal((H, d, d))
    scale = 0.3
    good = O.decode_sequence(q_nope, q_pe, c, kpe, w, w, scale)
    bad = O.decode_sequence(q_nope, q_pe, c, kpe, np.swapaxes(w, 1, 2), w, scale)
    assert np.max(np.abs(good - bad)) > 1e-3


# ------------------------------------------------------------------------
# 3. softmax rows
# ------------------------------------------------------------------------
def test_softmax_rows_sum_to_one_and_mask_is_exact():
    rng = _rng(5)
    H, sq, L = 3, 4, 10
    out, p = O.decode_sequence(rng.standard_normal((sq, H, 6)), rng.standard_normal((sq, H, 4)),
                               rng.standard_normal((L, 12)), rng.standard_normal((L, 4)),
                               rng.standard_normal((H, 6, 12)), rng.standard_normal((H, 5, 12)),
                               0.25, return_probs=True)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    for s in range(sq):
        last = L - sq + s
        assert np.all(p[s, :, last + 1:] == 0.0)
        assert np.all(p[s, :, : last + 1] > 0.0)


# ------------------------------------------------------------------------
# 4. special cases
# ------------------------------------------------------------------------
def _case(seed, H=3, dc=10, dr=4, dn=6, dv=5, L=8):
    rng = _rng(seed)
    return (rng.standard_normal((1, H, dn)), rng.standard_normal((1, H, dr)),
            rng.standard_normal((L, dc)), rng.standard_normal((L, dr)),
            rng.standard_normal((H, dn, dc)), rng.standard_normal((H, dv, dc)))


def test_single_token_is_its_value():
    qn, qp, c, kpe, wk, wv = _case(6, L=1)
    out = O.decode_sequence(qn, qp, c, kpe, wk, wv, 0.7)
    for h in range(wv.shape[0]):
        np.testing.assert_allclose(out[0, h], wv[h] @ c[0], rtol=1e-13)


def test_zero_query_gives_uniform_weights():
    qn, qp, c, kpe, wk, wv = _case(7)
    out = O.decode_sequence(0 * qn, 0 * qp, c, kpe, wk, wv, 0.7)
    for h in range(wv.shape[0]):
        np.testing.assert_allclose(out[0, h], wv[h] @ c.mean(0), rtol=1e-12)


def test_identical_rows_give_that_value():
    qn, qp, c, kpe, wk, wv = _case(8)
    c[:] = c[0]
    kpe[:] = kpe[0]
    out = O.decode_sequence(qn, qp, c, kpe, wk, wv, 0.7)
    for h in range(wv.shape[0]):
        np.testing.assert_allclose(out[0, h], wv[h] @ c[0], rtol=1e-12)


def test_rope_part_alone_can_select_a_token():
    """q_nope = 0: only q_pe . k_pe scores; a key aligned with q_pe dominates."""
    qn, qp, c, kpe, wk, wv = _case(9, H=1)
    kpe[:] = 0.0
    kpe[5] = 60.0 * qp[0, 0] / np.linalg.norm(qp[0, 0])
    out = O.decode_sequence(0 * qn, qp, c, kpe, wk, wv, 1.0)
    np.testing.assert_allclose(out[0, 0], wv[0] @ c[5], rtol=1e-12, atol=1e-12)


def test_nope_part_alone_can_select_a_token():
    """q_pe = 0: the score runs through W_UK; make token 2's latent dominate."""
    qn, qp, c, kpe, wk, wv = _case(10, H=1)
    direction = wk[0].T @ qn[0, 0]  # score_t = q_nope . (W_UK c_t) = (W_UK^T q_nope) . c_t
    c[2] = 80.0 * direction / np.linalg.norm(direction) ** 2
    out = O.decode_sequence(qn, 0 * qp, c, kpe, wk, wv, 1.0)
    np.testing.assert_allclose(out[0, 0], wv[0] @ c[2], rtol=1e-10, atol=1e-10)


def test_masked_spike_is_ignored():
    qn, qp, c, kpe, wk, wv = _case(11, L=9)
    qn = np.repeat(qn, 3, axis=0)
    qp = np.repeat(qp, 3, axis=0)
    base = O.decode_sequence(qn, qp, c, kpe, wk, wv, 0.5)
    c2, k2 = c.copy(), kpe.copy()
    c2[-1] *= 1e3  # visible only to the last new token
    k2[-1] = 1e3
    spiked = O.decode_sequence(qn, qp, c2, k2, wk, wv, 0.5)
    np.testing.assert_array_equal(spiked[:2], base[:2])
    assert np.max(np.abs(spiked[2] - base[2])) > 1e-6  # the last new token does see it


# ------------------------------------------------------------------------
# 5. textbook reduction: identity up-projections give plain SDPA
# ------------------------------------------------------------------------
@pytest.mark.parametrize("square", [True, False])
def test_identity_projections_reduce_to_sdpa(square):
    rng = _rng(12)
    H, dc, dr = 4, 16, 8
    L = 12
    sq = L if square else 1
    q_nope = rng.standard_normal((sq, H, dc))
    q_pe = rng.standard_normal((sq, H, dr))
    c = rng.standard_normal((L, dc))
    kpe = rng.standard_normal((L, dr))
    eye = np.stack([np.eye(dc)] * H)
    scale = 1.0 / math.sqrt(dc + dr)
    out = O.decode_sequence(q_nope, q_pe, c, kpe, eye, eye, scale)
    q = torch.from_numpy(np.concatenate([q_nope, q_pe], -1)).permute(1, 0, 2)  # [H, sq, d]
    k = torch.from_numpy(np.concatenate([c, kpe], -1))[None].expand(H, L, dc + dr)
    v = torch.from_numpy(c)[None].expand(H, L, dc)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=square, scale=scale)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------
# 6. RoPE
# ------------------------------------------------------------------------
def test_rope_matches_complex_rotation():
    """Rotate-half RoPE == complex multiply of pairs (x_i, x_{i+d/2}) by e^{i pos theta_i}."""
    rng = _rng(13)
    d = 64
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 17, 4095, 16383])
    got = O.rope(x, pos)
    z = x[:, : d // 2] + 1j * x[:, d // 2:]
    theta = np.array([10000.0 ** (-2.0 * i / d) for i in range(d // 2)])
    zr = z * np.exp(1j * pos[:, None] * theta[None])
    np.testing.assert_allclose(got, np.concatenate([zr.real, zr.imag], -1), rtol=1e-12, atol=1e-12)


def test_rope_hand_values():
    # d = 2: theta_0 = 1, so position 1 rotates (1, 0) by one radian.
    np.testing.assert_allclose(O.rope(np.array([1.0, 0.0]), 1), [math.cos(1), math.sin(1)], rtol=1e-15)
    # d = 4: theta_1 = 10000^(-1/2) = 0.01 rotates the (x1, x3) pair.
    got = O.rope(np.array([0.0, 1.0, 0.0, 0.0]), 100)
    np.testing.assert_allclose(got, [0.0, math.cos(1.0), 0.0, math.sin(1.0)], atol=1e-12)


def test_rope_invariants():
    rng = _rng(14)
    d = 64
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    np.testing.assert_array_equal(O.rope(q, 0), q)
    for p in (1, 300, 16380):
        assert abs(np.linalg.norm(O.rope(q, p)) - np.linalg.norm(q)) < 1e-12
    a = O.rope(q, 1000) @ O.rope(k, 990)
    b = O.rope(q, 10) @ O.rope(k, 0)
    assert abs(a - b) < 1e-9  # depends on m - n only


# ------------------------------------------------------------------------
# 7. RMSNorm
# ------------------------------------------------------------------------
def test_rmsnorm_closed_forms():
    a, eps = 3.0, 1e-6
    np.testing.assert_allclose(O.rmsnorm(np.full(8, a), eps=eps), a / math.sqrt(a * a + eps), rtol=1e-15)
    rng = _rng(15)
    v = rng.standard_normal((4, 512))
    out = O.rmsnorm(v, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, -1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rmsnorm(7.5 * v, eps=0.0), out, rtol=1e-13)
    g = rng.standard_normal(512)
    np.testing.assert_allclose(O.rmsnorm(v, g, eps=0.0), out * g, rtol=1e-13)


# ------------------------------------------------------------------------
# 8. split-KV combine
# ------------------------------------------------------------------------
def test_combine_of_any_partition_equals_unsplit():
    rng = _rng(16)
    L, dc, dr = 37, 24, 8
    q_lat, q_pe = rng.standard_normal(dc), rng.standard_normal(dr)
    c, kpe = rng.standard_normal((L, dc)), rng.standard_normal((L, dr))
    full_o, full_lse = O.latent_partial(q_lat, q_pe, c, kpe, 0.4)
    for cuts in ([0, 37], [0, 10, 37], [0, 1, 2, 20, 36, 37], [0, 0, 5, 5, 37, 37]):
        parts = [O.latent_partial(q_lat, q_pe, c[a:b], kpe[a:b], 0.4) for a, b in zip(cuts, cuts[1:])]
        o, lse = O.merge_partials(np.stack([p[0] for p in parts]), np.array([p[1] for p in parts]))
        np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-14)
        assert abs(lse - full_lse) < 1e-12


def test_combine_lse_matches_library_logsumexp():
    from scipy.special import logsumexp

    rng = _rng(17)
    z = rng.standard_normal(50) * 5
    c = rng.standard_normal((50, 3))
    _, lse = O.latent_partial(np.zeros(3), np.zeros(0), c * 0, np.zeros((50, 0)), 1.0)
    assert abs(lse - math.log(50)) < 1e-12
    # partial lse over halves merges to logsumexp of the whole
    lse_parts = np.array([logsumexp(z[:20]), logsumexp(z[20:])])
    _, m = O.merge_partials(np.zeros((2, 1)), lse_parts)
    assert abs(m - logsumexp(z)) < 1e-12


def test_combine_empty_partitions():
    o = np.array([[1.0, 2.0], [5.0, 5.0], [3.0, -1.0]])
    lse = np.array([-math.inf, 0.5, -math.inf])
    m, l = O.merge_partials(o, lse)
    np.testing.assert_array_equal(m, [5.0, 5.0])
    assert l == 0.5
    m, l = O.merge_partials(o, np.full(3, -math.inf))
    np.testing.assert_array_equal(m, [0.0, 0.0])
    assert l == -math.inf


# ------------------------------------------------------------------------
# 9. paging
# ------------------------------------------------------------------------
def test_resolve_slot_against_enumeration():
    bs = 64
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    lengths = I.context_lengths(w)
    table, total = I.block_table(w, lengths)
    owner = {}
    for b in range(w.batch):
        for j in range((int(lengths[b]) + bs - 1) // bs):
            blk = int(table[b, j])
            assert blk not in owner
            owner[blk] = (b, j)
    assert len(owner) == total
    for b in (0, 17, 63):
        for t in (0, 63, 64, int(lengths[b]) - 1):
            row = O.resolve_slot(table.numpy(), b, t, bs)
            blk, off = divmod(row, bs)
            assert owner[blk] == (b, t // bs) and off == t % bs


def test_contiguous_table_is_identity():
    w = I.WORKLOADS["tiny_b1_l128"]
    table, _ = I.block_table(w, I.context_lengths(w))
    assert [O.resolve_slot(table.numpy(), 0, t, 128) for t in range(128)] == list(range(128))


def test_gather_sequence_reads_rows_in_token_order():
    d = _small_dims(bs=4)
    nb = 5
    pool = np.zeros((nb, 4, d.row_width))
    for blk in range(nb):
        for off in range(4):
            pool[blk, off, :] = blk * 100 + off
    table = np.array([[2, 4, 0]])
    c, kpe = O.gather_sequence(pool, table, 0, 10, d)
    expect = [2 * 100 + t if t < 4 else (400 + t - 4 if t < 8 else t - 8) for t in range(10)]
    np.testing.assert_array_equal(c[:, 0], expect)
    np.testing.assert_array_equal(kpe[:, -1], expect)


# ------------------------------------------------------------------------
# 10. append chain invariants
# ------------------------------------------------------------------------
def test_append_chain_invariants():
    rng = _rng(18)
    x = rng.standard_normal((6, 32))
    w = rng.standard_normal((32, 24))
    pos = np.array([0, 0, 3, 10, 100, 16383])
    rows = O.append_rows(x, w, pos, 16, eps=0.0)
    kv = x @ w
    np.testing.assert_allclose(np.sqrt(np.mean(rows[:, :16] ** 2, -1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(rows[:, 16:], axis=-1), np.linalg.norm(kv[:, 16:], axis=-1),
                               rtol=1e-13)
    np.testing.assert_allclose(rows[:2, 16:], kv[:2, 16:], rtol=1e-14)  # position 0 = no rotation


def test_query_projection_head_layout():
    """A one-hot W_qb column lands in exactly one (head, index) of q_nope or q_pe:
    heads are the outer index of each row and the non-RoPE part comes first
    (a transposed view or a swapped split fails)."""
    H, dn, dr, R = 3, 4, 2, 8
    x = np.array([[1.0, -1, 1, 1, -1, 1, -1, -1], [-1.0, 1, 1, -1, 1, 1, 1, -1]])  # RMS 1 per row
    w_qa = np.eye(R)
    for h, j, r in [(0, 0, 3), (1, 2, 0), (2, 5, 7), (0, 4, 1), (2, 3, 6)]:
        w_qb = np.zeros((R, H * (dn + dr)))
        w_qb[r, h * (dn + dr) + j] = 1.0
        qn, qp = O.query_projection(x, w_qa, w_qb, np.zeros(2, dtype=int), H, dn, dr, eps=0.0)
        assert qn.shape == (2, H, dn) and qp.shape == (2, H, dr)
        want_n, want_p = np.zeros_like(qn), np.zeros_like(qp)
        if j < dn:
            want_n[:, h, j] = x[:, r]
        else:
            want_p[:, h, j - dn] = x[:, r]
        np.testing.assert_array_equal(qn, want_n)
        np.testing.assert_array_equal(qp, want_p)


def test_query_projection_matches_library_layers():
    """Against torch's own linear and rms_norm layers (float64): the non-RoPE part
    everywhere and the RoPE part at position 0 (no rotation) agree to rounding;
    at other positions each rotate-half pair keeps its norm."""
    rng = _rng(21)
    T, hid, R, H, dn, dr = 5, 24, 16, 3, 6, 4
    x = rng.standard_normal((T, hid))
    w_qa, w_qb = rng.standard_normal((hid, R)), rng.standard_normal((R, H * (dn + dr)))
    gamma = rng.uniform(0.5, 1.5, R)
    tx = torch.tensor(x)
    c = torch.nn.functional.rms_norm(torch.nn.functional.linear(tx, torch.tensor(w_qa.T)), (R,),
                                     weight=torch.tensor(gamma), eps=1e-6)
    q = torch.nn.functional.linear(c, torch.tensor(w_qb.T)).reshape(T, H, dn + dr).numpy()
    qn, qp0 = O.query_projection(x, w_qa, w_qb, np.zeros(T, dtype=int), H, dn, dr, gamma=gamma)
    np.testing.assert_allclose(qn, q[..., :dn], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(qp0, q[..., dn:], rtol=1e-12, atol=1e-12)
    pos = np.array([1, 7, 100, 4096, 16383])
    qn2, qp = O.query_projection(x, w_qa, w_qb, pos, H, dn, dr, gamma=gamma)
    np.testing.assert_array_equal(qn2, qn)  # the position touches only the RoPE part
    half = dr // 2
    np.testing.assert_allclose(np.hypot(qp[..., :half], qp[..., half:]), np.hypot(qp0[..., :half], qp0[..., half:]),
                               rtol=1e-12)
    assert not np.allclose(qp, qp0)
    # the rotation angle of pair i is position * base^(-2i/d_r)
    ang = pos[:, None, None] * O.rope_inv_freq(dr)[None, None, :]
    z0 = qp0[..., :half] + 1j * qp0[..., half:]
    np.testing.assert_allclose(qp[..., :half] + 1j * qp[..., half:], z0 * np.exp(1j * ang), rtol=1e-11, atol=1e-11)


def test_query_projection_is_scale_free_in_x():
    """The RMSNorm after q_a_proj makes the queries independent of the scale of x (eps = 0)."""
    rng = _rng(22)
    x = rng.standard_normal((3, 16))
    w_qa, w_qb = rng.standard_normal((16, 8)), rng.standard_normal((8, 2 * 6))
    a = O.query_projection(x, w_qa, w_qb, np.array([0, 5, 9]), 2, 4, 2, eps=0.0)
    b = O.query_projection(37.5 * x, w_qa, w_qb, np.array([0, 5, 9]), 2, 4, 2, eps=0.0)
    for u, v in zip(a, b):
        np.testing.assert_allclose(u, v, rtol=1e-12)


# ------------------------------------------------------------------------
# 11. the pages' printed structural numbers
# ------------------------------------------------------------------------
def test_dims_match_printed_sizes():
    import json
    import os

    with open(os.path.join(os.path.dirname(__file__), "golden", "v3_dims.json")) as f:
        g = json.load(f)
    d = I.V3
    assert d.row_width == g["cache_values_per_token"]
    assert d.num_heads * (d.qk_nope_dim + d.v_head_dim) == g["kv_b_proj_out"]
    assert (2 * d.num_heads * d.qk_nope_dim) // d.kv_lora_rank == g["latent_compression_ratio"]
    assert d.qk_nope_dim + d.rope_dim == g["qk_head_dim"]
    assert d.num_heads * (d.qk_nope_dim + d.rope_dim) == g["q_b_proj_out"]


# ------------------------------------------------------------------------
# output projection and W_UV absorbed into it
# ([MQA-MLA] "MLA的实现": forward_training's w_o and forward_inference_absorbed's
# W_o_absorbed = W_UV^T W_O; [MLA-arch] 3.1, W_V absorbed into the O projection)
# ------------------------------------------------------------------------
def _brute_output_projection(out, w_o):
    """y[t][m] = sum over heads h and value indices d of out[t][h][d] W_O[h d_v + d][m]."""
    T, H, dv = len(out), len(out[0]), len(out[0][0])
    hidden = len(w_o[0])
    y = [[0.0] * hidden for _ in range(T)]
    for t in range(T):
        for m in range(hidden):
            acc = 0.0
            for h in range(H):
                for d in range(dv):
                    acc += out[t][h][d] * w_o[h * dv + d][m]
            y[t][m] = acc
    return y


def test_output_projection_against_brute_force():
    rng = _rng(21)
    out = rng.standard_normal((3, 4, 5))
    w_o = rng.standard_normal((20, 7))
    np.testing.assert_allclose(O.output_projection(out, w_o), _brute_output_projection(out.tolist(), w_o.tolist()),
                               rtol=1e-12, atol=1e-12)


def test_output_projection_with_identity_weight_concatenates_heads():
    rng = _rng(22)
    out = rng.standard_normal((2, 3, 4))
    y = O.output_projection(out, np.eye(12))
    np.testing.assert_array_equal(y, out.reshape(2, 12))
    # one head's block alone: y reads that head's values only
    w = np.zeros((12, 4))
    w[4:8] = np.eye(4)
    np.testing.assert_array_equal(O.output_projection(out, w), out[:, 1, :])


@pytest.mark.parametrize("H,dc,dv,hidden", [(3, 8, 4, 5), (4, 32, 16, 24)])
def test_absorbed_output_weight_identity(H, dc, dv, hidden):
    """o_lat . (W_UV^T W_O) == (W_UV o_lat) . W_O for every head (associativity)."""
    rng = _rng(23)
    o_lat = rng.standard_normal((2, 3, H, dc))
    w_uv = rng.standard_normal((H, dv, dc)) / math.sqrt(dc)
    w_o = rng.standard_normal((H * dv, hidden))
    unfused = O.output_projection(O.up_project(o_lat, w_uv), w_o)
    fused = o_lat.reshape(2, 3, H * dc) @ O.absorbed_output_weight(w_uv, w_o)
    np.testing.assert_allclose(fused, unfused, rtol=1e-10, atol=1e-12)


def test_absorbed_output_weight_detects_head_mixups():
    """The identity is sharp: pairing head h's W_UV with another head's W_O block,
    or using W_UV without the transpose, breaks it."""
    rng = _rng(24)
    H, dc, dv, hidden = 3, 6, 6, 5
    o_lat = rng.standard_normal((4, H, dc))
    w_uv = rng.standard_normal((H, dv, dc))
    w_o = rng.standard_normal((H * dv, hidden))
    good = O.output_projection(O.up_project(o_lat, w_uv), w_o)
    rolled = O.absorbed_output_weight(np.roll(w_uv, 1, axis=0), w_o)
    untransposed = np.concatenate([w_uv[h] @ w_o[h * dv:(h + 1) * dv] for h in range(H)], axis=0)
    for bad_w in (rolled, untransposed):
        assert np.max(np.abs(o_lat.reshape(4, H * dc) @ bad_w - good)) > 1e-3


def test_decode_latent_up_projects_to_the_explicit_decode():
    """W_UV applied to the latent decode output equals the explicit
    (decompressed) decode, over a paged pool with several new tokens."""
    rng = _rng(25)
    d = _small_dims(H=3, dc=8, dr=4, dn=5, dv=4, bs=4)
    lengths = [9, 4]
    sq = 2
    table = np.array([[5, 1, 3], [0, -1, -1]])
    pool = rng.standard_normal((6, d.block_size, d.row_width))
    q_nope = rng.standard_normal((2, sq, d.num_heads, d.qk_nope_dim))
    q_pe = rng.standard_normal((2, sq, d.num_heads, d.rope_dim))
    w_uk = rng.standard_normal((d.num_heads, d.qk_nope_dim, d.kv_lora_rank))
    w_uv = rng.standard_normal((d.num_heads, d.v_head_dim, d.kv_lora_rank))
    scale = 0.4
    o_lat = O.decode_latent_paged(q_nope, q_pe, pool, table, lengths, w_uk, d, scale)
    explicit = O.decode_paged(q_nope, q_pe, pool, table, lengths, w_uk, w_uv, d, scale)
    np.testing.assert_allclose(O.up_project(o_lat, w_uv), explicit, rtol=1e-10, atol=1e-12)
