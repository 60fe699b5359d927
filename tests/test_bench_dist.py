"""Multi-process host logic of bench.py on CPU (gloo, world size 2): each rank
gets its own replica seed, the step time reported is the max over ranks, and
the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    dist = bench.init_dist("gloo", world, timeout_s=60)
    r, w, lr = bench.dist_env()
    seed = bench.rank_seed(1002, r)
    t = bench.max_over_ranks(1.0 + 2.0 * r, "cpu")
    bench.barrier()
    q.put((r, w, seed, t))
    dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert res[0][2] != res[1][2]  # distinct replicas
    assert all(r[3] == 3.0 for r in res)  # max over ranks


def test_reference_arm_only_on_rank_zero(monkeypatch):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 1, "warmup": 3})()
    from mla_latent_kv_29_b200 import inputs as I

    assert bench.run_reference(args, I.WORKLOADS["v3_b64_l1k_8k"]) is None


def test_workload_totals_counts_units():
    import bench
    from mla_latent_kv_29_b200 import inputs as I

    w = I.scaled(I.WORKLOADS["v3_b16_sq4_l16k_append"], batch=2, length=100)
    t = bench.workload_totals(w, [100, 10])
    assert t["T"] == 110
    assert t["V"] == (97 + 98 + 99 + 100) + (7 + 8 + 9 + 10)
    assert t["attn_bytes"] == 110 * 1152 + 8 * 128 * 1152
    assert t["attn_flops"] == 2 * 128 * (576 + 512) * t["V"]
