"""Host arithmetic of bench.py on CPU: the algorithmic units the roofline
divides by, the bound selection and the recorded-traffic guard."""
import dataclasses

import bench
from mla_latent_kv_29_b200 import inputs as I


def test_attention_units_by_hand():
    """Two sequences of 3 and 5 tokens, two new tokens each, V3 dims."""
    w = dataclasses.replace(I.WORKLOADS["v3_b64_l1k_8k"], batch=2, q_len=2)
    tot = bench.workload_totals(w, [3, 5])
    assert tot["T"] == 8
    # visible pairs: (3: 2, 3) + (5: 4, 5)
    assert tot["V"] == 2 + 3 + 4 + 5
    assert tot["G"] == 4
    assert tot["attn_bytes"] == 8 * 1152 + 4 * 128 * 1152
    assert tot["attn_flops"] == 2 * 128 * (576 + 512) * 14


def test_roofline_picks_the_slower_bound():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    r, gbs, tfs = bench.roofline(1e9, 1e10, 2e-3, peaks)  # 1 ms of bytes, 0.1 ms of flops
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["frac"] - 0.5) < 1e-12
    r, _, _ = bench.roofline(1e6, 1e12, 20e-3, peaks)  # 1 us of bytes, 10 ms of flops
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and abs(r["frac"] - 0.5) < 1e-12


def test_q_proj_units():
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    line = bench.q_proj_line(w, 0.1, {"hbm_gbs": 6538.0})
    assert line["bytes"] == 2 * (7168 * 1536 + 1536 * 128 * 192 + 64 * 7168 + 64 * 128 * 192)
    assert line["tokens"] == 64
    assert abs(line["achieved_gbs"] - line["bytes"] / 1e-4 / 1e9) < 0.1


def test_traffic_is_reported_only_for_the_recorded_sources():
    rec = bench.TRAFFIC["v3_b64_l1k_8k"]
    if bench.kernel_sources_sha256() == rec["sources_sha256"]:
        assert bench.recorded_traffic("v3_b64_l1k_8k") == rec["bytes"]
    else:
        assert bench.recorded_traffic("v3_b64_l1k_8k") is None
    assert bench.recorded_traffic("no_such_workload") is None


def test_both_arms_share_the_workload_config():
    w = I.WORKLOADS["v3_b64_l1k_8k"]
    c = bench.workload_config(w, 274358)
    assert c["workload"] == "v3_b64_l1k_8k" and c["batch_per_gpu"] == 64 and c["paged"] == "shuffled"
    assert c["cached_tokens_per_gpu"] == 274358
