#!/usr/bin/env python
"""Benchmark of one MLA absorbed-decode step on B200.

A step is one pass of the whole hot path over one batch: the cache append of
the batch's new tokens (down-projection, RMSNorm, RoPE, paged write) and the
absorbed decode of those tokens (query absorption, split-KV attention over
the paged latent cache, log-sum-exp combine, value up-projection).

Default workload: DeepSeek-V3 shapes (128 heads, latent 512 + RoPE 64),
batch 64, one new token per sequence, context lengths uniform in
[1024, 8192], 64-token pages with a shuffled block table. The cache is filled
before timing by the library's own append from x ~ N(0,1) hidden states and
a kv_a weight ~ N(0, 1/7168), so every row is an RMS-normalised latent plus
a RoPE-rotated key, as the workload prescribes.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs its own replica (independent batches,
no collective on the data path): weak scaling, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MLA absorbed decode µs/step, cache GB/s & TFLOPS as fraction of B200 roofline"
UNIT = "µs/step"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
L2_FLUSH_BYTES = 256 << 20
HIDDEN = 7168


# ----------------------------------------------------------- distributed
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(backend: str, world: int, timeout_s: float = 120.0):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def rank_seed(base: int, rank: int) -> int:
    """Each rank's replica draws its own batch."""
    return base + 7919 * rank


def max_over_ranks(value: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------- roofline
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS)


STEP_TEXT = "append of the batch's new tokens + absorbed decode"


def workload_config(w, cached_tokens):
    """The workload's identity: the same object in both arms' lines (how each
    arm times it goes in its own `timing` entry)."""
    return {"workload": w.name, "batch_per_gpu": w.batch, "q_len": w.q_len,
            "context": f"U[{w.length_range[0]},{w.length_range[1]}]", "cached_tokens_per_gpu": cached_tokens,
            "heads": w.dims.num_heads, "latent": w.dims.kv_lora_rank, "rope": w.dims.rope_dim,
            "page": w.dims.block_size, "paged": "shuffled" if w.paged else "contiguous", "step": STEP_TEXT}


def spread(values_ms):
    """median / p10 / p90 (µs) of per-step times given in ms."""
    v = sorted(values_ms)
    q = lambda f: v[min(len(v) - 1, max(0, int(round(f * (len(v) - 1)))))]
    return {"reps": len(v), "median_us": round(statistics.median(v) * 1e3, 2), "p10_us": round(q(0.1) * 1e3, 2),
            "p90_us": round(q(0.9) * 1e3, 2), "mean_us": round(statistics.mean(v) * 1e3, 2)}


def workload_totals(w, lengths):
    """Algorithmic units of one decode step. Attention: every cached token's
    576 bf16 values read once plus the absorbed queries; FLOPs 2 H (576 + 512)
    per visible (query, token) pair. Step: the attention's cache bytes, the
    W_UK / W_UV / W_kva weights, the new tokens' inputs and the outputs."""
    d = w.dims
    L = [int(v) for v in lengths]
    T = sum(L)  # unique cached tokens read
    V = sum(Lb - w.q_len + s + 1 for Lb in L for s in range(w.q_len))  # visible (query, token) pairs
    G = w.batch * w.q_len
    row = d.row_width * 2  # bytes per cached token
    attn_bytes = T * row + G * d.num_heads * row  # cache rows + absorbed queries
    # FP8 cache: d_c codes + d_r f16 + one fp32 scale per token (644 bytes for V3)
    attn_bytes_fp8 = T * (d.kv_lora_rank + 2 * d.rope_dim + 4) + G * d.num_heads * row
    attn_flops = 2 * d.num_heads * (d.row_width + d.kv_lora_rank) * V
    w_bytes = 2 * d.num_heads * (d.qk_nope_dim + d.v_head_dim) * d.kv_lora_rank * 2
    step_bytes = T * row + w_bytes + G * d.num_heads * (d.qk_nope_dim + d.rope_dim + d.v_head_dim) * 2
    step_flops = attn_flops + 2 * G * d.num_heads * (d.qk_nope_dim + d.v_head_dim) * d.kv_lora_rank
    # every step appends its G new tokens (x [G, 7168] times W_kva [7168, 576])
    step_bytes += HIDDEN * d.row_width * 2 + G * HIDDEN * 2
    step_flops += 2 * G * HIDDEN * d.row_width
    return dict(T=T, V=V, G=G, attn_bytes=attn_bytes, attn_flops=attn_flops, step_bytes=step_bytes,
                step_flops=step_flops, attn_bytes_fp8=attn_bytes_fp8)


Q_RANK = 1536  # q_lora_rank of the DeepSeek-V3 query path


def q_proj_line(w, ms, peaks):
    """Roofline of mla_q_proj for the step's G new tokens: bytes = W_qa + W_qb +
    x + q_nope + q_pe (bf16); FLOPs = 2 G (hidden q_rank + q_rank H (d_n + d_r))."""
    d = w.dims
    G = w.batch * w.q_len
    n2 = d.num_heads * (d.qk_nope_dim + d.rope_dim)
    bytes_ = 2 * (HIDDEN * Q_RANK + Q_RANK * n2 + G * HIDDEN + G * n2)
    flops = 2 * G * (HIDDEN * Q_RANK + Q_RANK * n2)
    gbs = bytes_ / (ms * 1e-3) / 1e9
    return {"us": round(ms * 1e3, 2), "tokens": G, "hidden": HIDDEN, "q_rank": Q_RANK,
            "bytes": bytes_, "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
            "frac": round(gbs / peaks["hbm_gbs"], 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "timing": "CUDA events around each call, L2 flushed before each, K calls"}


def roofline(bytes_, flops, seconds, peaks):
    """The bound whose time is larger, against the given peaks; `frac_nominal`
    is the same achieved figure against the nominal B200 peaks (8 TB/s HBM,
    2.25 PFLOP/s dense bf16), the roofline the target is stated on."""
    gbs = bytes_ / seconds / 1e9
    tfs = flops / seconds / 1e12
    t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    # the other bound too: the absorbed decode sits near the ridge, where both matter
    frac_hbm, frac_tc = round(gbs / peaks["hbm_gbs"], 4), round(tfs / peaks["bf16_tflops"], 4)
    if t_hbm >= t_tc:
        return dict(bound="hbm", achieved=round(gbs, 1), peak=peaks["hbm_gbs"], unit="GB/s", frac=frac_hbm,
                    frac_nominal=round(gbs / NOMINAL["hbm_gbs"], 4), peak_nominal=NOMINAL["hbm_gbs"],
                    other_bound={"bound": "tensor", "achieved": round(tfs, 2), "peak": peaks["bf16_tflops"],
                                 "unit": "TFLOP/s", "frac": frac_tc}), gbs, tfs
    return dict(bound="tensor", achieved=round(tfs, 2), peak=peaks["bf16_tflops"], unit="TFLOP/s", frac=frac_tc,
                frac_nominal=round(tfs / NOMINAL["bf16_tflops"], 4), peak_nominal=NOMINAL["bf16_tflops"],
                other_bound={"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": frac_hbm}), gbs, tfs


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the attention kernel from an ncu capture of this bench's workload, valid only
# for the kernel sources it was taken on (their SHA-256 below; the capture and
# its command are summarised under profiles/). Any change to those sources
# turns the reported traffic into null until a new capture is recorded here.
KERNEL_SOURCES = ("decode_pair.cuh", "plan.cuh", "sm100.cuh", "common.cuh", "fp8.cuh")
TRAFFIC = {
    # profiles/pair_decode_kernel_v3_b64_l1k_8k.md (ncu launch list of one step, the attention launch:
    # dram__bytes_read.sum + dram__bytes_write.sum)
    "v3_b64_l1k_8k": {"bytes": 364470016 + 6244096,
                      "sources_sha256": "baeea80604bb1b037e1d8110b71db95da3e8396156de9ed42264571c4c8de60e"},
}

def kernel_sources_sha256() -> str:
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mla_latent_kv_29_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    rec = TRAFFIC.get(workload)
    if rec is None or rec["sources_sha256"] != kernel_sources_sha256():
        return None
    return rec["bytes"]


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(period_ms), "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------- CPU (oracle)
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_seconds(w, lengths, seqs, heads):
    """Times the fp64 oracle (explicit decode + append rows) on a few sequences and heads.

    Inputs are drawn on the host from the same seeded generators (the
    oracle never reads device data); only the timed calls are the oracle's.
    """
    import numpy as np

    from mla_latent_kv_29_b200 import inputs as I
    from oracle import mla_oracle as O

    d = w.dims
    q_nope, q_pe = I.queries(w)
    w_uk, w_uv = I.up_weights(w)
    x_new = I.normal((w.q_len, HIDDEN), 1.0, w.seed, 7)
    w_kva = I.normal((HIDDEN, d.row_width), HIDDEN ** -0.5, w.seed, 8)
    total = 0.0
    tokens = 0
    for b in seqs:
        L = int(lengths[b])
        c_raw, pe_raw = I.cache_raw(w, b, L)
        c = O.rmsnorm(c_raw)
        kpe = O.rope(pe_raw, np.arange(L))
        qn = I.bf16(q_nope[b][:, heads]).double().numpy()
        qp = I.bf16(q_pe[b][:, heads]).double().numpy()
        wk = I.bf16(w_uk[heads]).double().numpy()
        wv = I.bf16(w_uv[heads]).double().numpy()
        t0 = time.perf_counter()
        O.append_rows(x_new, w_kva, np.arange(L - w.q_len, L), d.kv_lora_rank)
        O.decode_sequence(qn, qp, c, kpe, wk, wv, w.softmax_scale)
        total += time.perf_counter() - t0
        tokens += L
    return total, tokens


def cpu_baseline(w, lengths, budget_s: float = 12.0):
    """Oracle µs/step for the whole workload, extrapolated from a bounded sample."""
    H = w.dims.num_heads
    heads = list(range(0, H, 4))  # a quarter of the heads
    T = sum(int(v) for v in lengths)
    spent, tok, seqs = 0.0, 0, []
    for b in range(w.batch):
        s, t = oracle_sample_seconds(w, lengths, [b], heads)
        spent += s
        tok += t
        seqs.append(b)
        if spent >= budget_s:
            break
    per_step_s = spent * (T / tok) * (H / len(heads))
    return {"value": round(per_step_s * 1e6, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 explicit oracle on {len(seqs)} of {w.batch} sequences ({tok} of {T} cached "
                      f"tokens), {len(heads)} of {H} heads, plus their append rows; scaled by tokens and "
                      f"heads to the full step ({spent:.1f} s measured)"}


# -------------------------------------------------------------- GPU leg
def setup_gpu(w, device, rank):
    import torch

    from mla_latent_kv_29_b200 import inputs as I
    from mla_latent_kv_29_b200 import lib

    d = w.dims
    lengths = I.context_lengths(w)
    table, nblk = I.block_table(w, lengths)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    pool = torch.empty(nblk, d.block_size, d.row_width, dtype=torch.bfloat16, device=device)
    table_d = table.to(device)
    w_kva = (torch.randn(HIDDEN, d.row_width, generator=gen, device=device) * HIDDEN ** -0.5).to(torch.bfloat16)
    # fill positions 0 .. L_b - q_len - 1 of every sequence through the library's append
    seq_ids = torch.cat([torch.full((int(L) - w.q_len,), b, dtype=torch.int32) for b, L in enumerate(lengths)])
    pos = torch.cat([torch.arange(int(L) - w.q_len, dtype=torch.int32) for L in lengths])
    chunk = 16384
    ws = torch.empty(lib.append_workspace_size(d, chunk, HIDDEN) + 256, dtype=torch.uint8, device=device)
    for i in range(0, seq_ids.numel(), chunk):
        n = min(chunk, seq_ids.numel() - i)
        x = torch.randn(n, HIDDEN, generator=gen, device=device).to(torch.bfloat16)
        lib.append_kv(d, x, w_kva, seq_ids[i:i + n].to(device), pos[i:i + n].to(device), table_d, pool,
                      workspace=ws)
    torch.cuda.synchronize(device)
    assert lib.device_error() == 0
    G = w.batch * w.q_len
    new_seq = torch.arange(w.batch, dtype=torch.int32).repeat_interleave(w.q_len)
    new_pos = (lengths.repeat_interleave(w.q_len) - w.q_len +
               torch.arange(w.q_len, dtype=torch.int32).repeat(w.batch)).to(torch.int32)
    st = dict(
        d=d, lengths=lengths, lengths_d=lengths.to(device), table=table_d, pool=pool, w_kva=w_kva,
        x_new=torch.randn(G, HIDDEN, generator=gen, device=device).to(torch.bfloat16),
        new_seq=new_seq.to(device), new_pos=new_pos.to(device),
        q_nope=torch.randn(w.batch, w.q_len, d.num_heads, d.qk_nope_dim, generator=gen, device=device).to(torch.bfloat16),
        q_pe=torch.randn(w.batch, w.q_len, d.num_heads, d.rope_dim, generator=gen, device=device).to(torch.bfloat16),
        w_uk=(torch.randn(d.num_heads, d.qk_nope_dim, d.kv_lora_rank, generator=gen, device=device) * w.w_std).to(torch.bfloat16),
        w_uv=(torch.randn(d.num_heads, d.v_head_dim, d.kv_lora_rank, generator=gen, device=device) * w.w_std).to(torch.bfloat16),
        out=torch.empty(w.batch, w.q_len, d.num_heads, d.v_head_dim, dtype=torch.bfloat16, device=device),
        max_len=int(lengths.max()),
    )
    st["ws_append"] = torch.empty(lib.append_workspace_size(d, G, HIDDEN) + 256, dtype=torch.uint8, device=device)
    st["ws_decode"] = torch.empty(lib.decode_workspace_size(d, w.softmax_scale, w.batch, w.q_len, st["max_len"]),
                                  dtype=torch.uint8, device=device)
    return st


def make_step(w, st, kernel, overlap=True, fp8=False):
    """One step: the append of the batch's new tokens, then the decode. With
    overlap the append runs on a side stream beside the decode's schedule and
    query absorption, and the decode's attention waits for it (cache_ready).
    fp8: both run on the FP8 cache st["pool8"] (mla_append_kv_fp8, and the
    decode with cache_fp8)."""
    import torch

    from mla_latent_kv_29_b200 import lib

    d = st["d"]
    side = torch.cuda.Stream() if overlap else None
    fork, ready = torch.cuda.Event(), torch.cuda.Event()
    fork.record()
    ready.record()  # the handles exist before any capture

    pool = st["pool8"] if fp8 else st["pool"]

    def append(x_new, stream=None):
        lib.append_kv(d, st["x_new"] if x_new is None else x_new, st["w_kva"], st["new_seq"], st["new_pos"],
                      st["table"], pool, workspace=st["ws_append"], stream=stream, fp8=fp8)

    def step(x_new=None, q_nope=None, q_pe=None, events=None):
        if side is not None:
            cur = torch.cuda.current_stream()
            fork.record(cur)
            side.wait_event(fork)
            append(x_new, stream=side)
            ready.record(side)
        else:
            append(x_new)
        lib.decode(d, w.softmax_scale, st["q_nope"] if q_nope is None else q_nope,
                   st["q_pe"] if q_pe is None else q_pe, pool, st["table"], st["lengths_d"], st["max_len"],
                   st["w_uk"], st["w_uv"], out=st["out"], workspace=st["ws_decode"], kernel=kernel,
                   attn_events=events, cache_ready=ready if side is not None else None, cache_fp8=fp8)

    return step


def count_library_launches(step, device):
    """Kernels of this library (names in the mla:: namespace) launched by one
    untimed step, as seen by the CUDA activity profiler."""
    import torch
    from torch.profiler import ProfilerActivity, profile

    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize(device)
    names = [e.name for e in prof.events() if "CUDA" in str(e.device_type) and "mla::" in e.name]
    return len(names), sorted(set(n.split("(")[0].replace("void ", "") for n in names))


def timed_calls(fn, flush, K, warmup, device):
    """Device times (ms) of K calls of fn, each after an L2 flush, CUDA events
    on the current stream."""
    import torch

    for _ in range(warmup):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize(device)
    for k in range(K):
        flush.zero_()
        ev[k][0].record()
        fn()
        ev[k][1].record()
    torch.cuda.synchronize(device)
    return [a.elapsed_time(b) for a, b in ev]


def o_proj_lines(w, st, flush, K, warmup, device, peaks):
    """The output projection of the step's G tokens, two ways (mla_o_proj):
    unfused, out [G, H d_v] times W_O [H d_v, 7168] after the per-head W_UV;
    absorbed, o_lat [G, H d_c] times W_UV^T W_O [H d_c, 7168] (the decode with
    output_latent). Weights are random of those shapes (the product's values
    do not change the traffic); bytes = weights + activations in + out."""
    import torch

    from mla_latent_kv_29_b200 import lib

    d = st["d"]
    G = w.batch * w.q_len
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 77)
    res = {}
    for name, k in (("unfused", d.num_heads * d.v_head_dim), ("absorbed", d.num_heads * d.kv_lora_rank)):
        wt = (torch.randn(k, HIDDEN, generator=gen, device=device) * k ** -0.5).to(torch.bfloat16)
        x = torch.randn(G, k, generator=gen, device=device).to(torch.bfloat16)
        y = torch.empty(G, HIDDEN, dtype=torch.bfloat16, device=device)
        ws = torch.empty(lib.o_proj_workspace_size(G, k, HIDDEN), dtype=torch.uint8, device=device)
        ms = timed_calls(lambda: lib.o_proj(x, wt, y=y, workspace=ws), flush, K, warmup, device)
        t = statistics.median(ms)
        bytes_ = 2 * (k * HIDDEN + G * k + G * HIDDEN)
        gbs = bytes_ / (t * 1e-3) / 1e9
        res[name] = {"us": round(t * 1e3, 2), "k": k, "n": HIDDEN, "tokens": G, "bytes": bytes_,
                     "achieved_gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4)}
        del wt, x, y, ws
    res["absorbed_over_unfused_time"] = round(res["absorbed"]["us"] / res["unfused"]["us"], 3)
    res["timing"] = "median of K calls, CUDA events around each, L2 flushed before each"
    return res


def workload_summary(name, args, device, peaks, flush, K=10, fp8=False):
    """Step and attention times of another workload (same step as the headline:
    append of the new tokens + decode, CUDA graph replay, L2 flushed before
    each step), for the summary of every configuration. fp8: the same step on
    the workload's cache converted to the FP8 format (mla_cache_to_fp8; the
    bf16 pool is freed), appending with mla_append_kv_fp8."""
    import dataclasses

    import torch

    from mla_latent_kv_29_b200 import inputs as I
    from mla_latent_kv_29_b200 import lib

    rank, _, _ = dist_env()
    w = I.WORKLOADS[name]
    w = dataclasses.replace(w, seed=rank_seed(w.seed, rank))
    st = setup_gpu(w, device, rank)
    if fp8:
        st["pool8"] = lib.cache_to_fp8(st["d"], st["pool"])
        st["pool"] = None
        torch.cuda.synchronize(device)
    step = make_step(w, st, args.kernel, overlap=args.overlap, fp8=fp8)
    ea = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ea[0].record()
    ea[1].record()
    graphs = []

    def capture(events):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(events=events)
        g.replay()
        torch.cuda.synchronize(device)
        graphs.append(g)
        return g.replay

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    run, run_attn = capture(None), capture(ea)
    step_ms = timed_calls(run, flush, K, 2, device)
    attn_ms = []
    for _ in range(K):
        flush.zero_()
        run_attn()
        torch.cuda.synchronize(device)
        attn_ms.append(ea[0].elapsed_time(ea[1]))
    tot = workload_totals(w, st["lengths"].tolist())
    t_attn = statistics.median(attn_ms) / 1e3
    attn_bytes = tot["attn_bytes_fp8"] if fp8 else tot["attn_bytes"]
    roof, gbs, tfs = roofline(attn_bytes, tot["attn_flops"], t_attn, peaks)
    assert lib.device_error() == 0
    del graphs, st
    torch.cuda.synchronize(device)
    return {"step_us_median": round(statistics.median(step_ms) * 1e3, 2),
            "attn_us_median": round(t_attn * 1e6, 2), "attn_bound": roof["bound"], "attn_frac": roof["frac"],
            "attn_frac_nominal": roof["frac_nominal"], "attn_gbs": round(gbs, 1), "attn_tflops": round(tfs, 2),
            "attn_bytes": attn_bytes, "cached_tokens": tot["T"], "new_tokens": tot["G"], "steps": K}


def run_ours(args, w):
    import torch

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist("nccl", world)
    from mla_latent_kv_29_b200 import inputs as I
    from mla_latent_kv_29_b200 import lib

    lib.load()
    st = setup_gpu(w, device, rank)
    step = make_step(w, st, args.kernel, overlap=args.overlap)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert lib.device_error() == 0, "device fault during warm-up"
    launches_per_step, kernel_names = count_library_launches(step, device)

    sampler = ClockSampler(device.index)
    soak_end = time.time() + args.soak
    while time.time() < soak_end:  # holds the GPU under the step's load while the sampler starts
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ea = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ea[0].record()
    ea[1].record()  # the handles exist before any capture
    # The timed region is K steps without timing events inside them: an event
    # recorded between two launches stands between them in the graph and takes
    # away their programmatic overlap. The attention kernel's time comes from a
    # second pass of K steps right after it, whose steps record events right
    # before and after its launch.
    def capture(events):
        if not args.graph:
            return lambda: step(events=events)
        g = torch.cuda.CUDAGraph()  # the step's launches replayed from one graph (no host launch gaps)
        with torch.cuda.graph(g):
            step(events=events)
        g.replay()
        torch.cuda.synchronize(device)
        graphs.append(g)
        return g.replay

    graphs = []
    run, run_attn = capture(None), capture(ea)
    ev_attn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    attn_ms = []
    barrier(device)
    torch.cuda.synchronize(device)
    for k in range(K):
        flush.zero_()  # evicts L2 (126 MB) between timed steps
        ev[k][0].record()
        run()
        ev[k][1].record()
    torch.cuda.synchronize(device)
    barrier(device)
    for k in range(K):  # the attention pass (after the timed region)
        flush.zero_()
        ev_attn[k][0].record()
        run_attn()
        ev_attn[k][1].record()
        ev_attn[k][1].synchronize()
        attn_ms.append(ea[0].elapsed_time(ea[1]))
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    step_ms_attn_pass = [a.elapsed_time(b) for a, b in ev_attn]
    assert lib.device_error() == 0, "device fault during the timed steps"

    # end to end through the public API with host buffers: the step's inputs sit
    # back to back in one pinned host buffer and cross to the device in one copy
    # (one copy instead of five: each copy has its own fixed cost); the step
    # reads them through device views of the staging buffer
    pieces = [st["x_new"], st["q_nope"], st["q_pe"], st["new_seq"], st["new_pos"]]
    offs, total = [], 0
    for t_ in pieces:
        offs.append(total)
        total += (t_.numel() * t_.element_size() + 255) // 256 * 256
    h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(total, dtype=torch.uint8, device=device)
    views = []
    for t_, o in zip(pieces, offs):
        n = t_.numel() * t_.element_size()
        h_in[o:o + n].copy_(t_.reshape(-1).view(torch.uint8).cpu())
        views.append(d_in[o:o + n].view(t_.dtype).view(t_.shape))
    d_x, d_qn, d_qp, d_seq, d_pos = views
    st["new_seq"], st["new_pos"] = d_seq, d_pos  # the e2e step's append reads its slots from the staging buffer
    h_out = torch.empty(st["out"].shape, dtype=torch.bfloat16).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e2e_graph = None
    if args.graph:
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph):
            step(x_new=d_x, q_nope=d_qn, q_pe=d_qp)
        torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    for k in range(K):
        flush.zero_()
        e2e_ev[k][0].record()
        d_in.copy_(h_in, non_blocking=True)
        if e2e_graph is not None:
            e2e_graph.replay()
        else:
            step(x_new=d_x, q_nope=d_qn, q_pe=d_qp)
        h_out.copy_(st["out"], non_blocking=True)
        e2e_ev[k][1].record()
    torch.cuda.synchronize(device)
    barrier(device)
    e2e_ms = [a.elapsed_time(b) for a, b in e2e_ev]
    t_e2e_pipe = e2e_pipelined(args, step, st, pieces, offs, total, h_in, K, device)

    t_step = max_over_ranks(statistics.mean(step_ms), device)
    t_attn = max_over_ranks(statistics.mean(attn_ms), device)
    # the query projection of the step's new tokens (mla_q_proj, a separate pass:
    # the decode above takes its queries as inputs), each call after an L2 flush
    d = st["d"]
    qin = I.q_proj_inputs(d, w.batch * w.q_len, HIDDEN, Q_RANK, seed=w.seed)
    qdev = {k: v.to(device) for k, v in qin.items()}
    q_ws = torch.empty(lib.q_proj_workspace_size(d, w.batch * w.q_len, HIDDEN, Q_RANK), dtype=torch.uint8,
                       device=device)
    q_out = (torch.empty_like(st["q_nope"]).view(-1, d.num_heads, d.qk_nope_dim),
             torch.empty_like(st["q_pe"]).view(-1, d.num_heads, d.rope_dim))

    def q_proj():
        lib.q_proj(d, qdev["x"], qdev["w_qa"], qdev["w_qb"], qdev["positions"], q_gamma=qdev["gamma"],
                   q_nope=q_out[0], q_pe=q_out[1], workspace=q_ws)

    for _ in range(args.warmup):
        q_proj()
    q_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize(device)
    for k in range(K):
        flush.zero_()
        q_ev[k][0].record()
        q_proj()
        q_ev[k][1].record()
    torch.cuda.synchronize(device)
    assert lib.device_error() == 0, "device fault in the query projection"
    t_q = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in q_ev), device)
    t_e2e = max_over_ranks(statistics.mean(e2e_ms), device)
    t_e2e_pipe = max_over_ranks(t_e2e_pipe, device)
    if rank != 0:
        return None
    tot = workload_totals(w, st["lengths"].tolist())
    peaks = load_peaks()
    roof, attn_gbs, attn_tfs = roofline(tot["attn_bytes"], tot["attn_flops"], t_attn / 1e3, peaks)
    roof["traffic"] = recorded_traffic(w.name) if args.kernel in (0, 1) else None
    roof["kernel"] = "split-KV attention" + (" (CUDA cores)" if args.kernel == 2 else "")
    roof["peak_source"] = peaks["source"]
    nominal_step = max(tot["step_bytes"] / (NOMINAL["hbm_gbs"] * 1e9), tot["step_flops"] / (NOMINAL["bf16_tflops"] * 1e12))
    line = {
        "metric": METRIC, "value": round(t_step * 1e3, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t_step, 5), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, tot["T"]),
        "timing": {"l2": "flushed (256 MB write) before each step",
                   "append": "on a side stream; the attention waits for it" if args.overlap else "in stream order",
                   "launch": "CUDA graph replay" if args.graph else "direct launches",
                   "value": "mean of the K device-timed steps (CUDA events on the launch stream), max over ranks",
                   "step_spread": spread(step_ms), "attn_spread": spread(attn_ms)},
        "roofline": roof,
        "attn_us": round(t_attn * 1e3, 2),
        "attn_timing": "CUDA events around the attention launch, in a second pass of K steps "
                       f"(step time in that pass {statistics.mean(step_ms_attn_pass) * 1e3:.2f} us)",
        "attn_hbm_gbs": round(attn_gbs, 1), "attn_tflops": round(attn_tfs, 2),
        "cache_tokens_per_s": round(world * tot["T"] / (t_step / 1e3), 1),
        "decode_tokens_per_s": round(world * tot["G"] / (t_step / 1e3), 1),
        "step_roofline_nominal_us": round(nominal_step * 1e6, 2),
        "step_frac_of_nominal_roofline": round(nominal_step / (t_step / 1e3), 4),
        "e2e": {"value": round(t_e2e_pipe * 1e3, 2), "unit": UNIT,
                "h2d_bytes_per_step": h_in.numel(),
                "d2h_bytes_per_step": h_out.numel() * 2,
                "timing": "K steps back to back through the public calls: each step copies its inputs from pinned "
                          "host memory and its output back; two staging and output buffers let step k's copies "
                          "overlap steps k - 1 and k + 1 (copy streams in, compute, copy streams out); total time / "
                          "K, no L2 flush between steps (the cache exceeds L2, but the layer's 42 MB of weights stay "
                          "in L2 from one step to the next, which is why this can come out below the flushed "
                          "device-timed step)",
                "serial_value": round(t_e2e * 1e3, 2),
                "serial_timing": "each step alone: L2 flush, copy in, step, copy out, CUDA events around the three"},
        "gpu_launches": launches_per_step * K,
        "q_proj": q_proj_line(w, t_q, peaks),
        "o_proj": o_proj_lines(w, st, flush, min(K, 20), args.warmup, device, peaks),
        "kernels": kernel_names,
        "clocks": clocks,
    }
    if args.all_workloads:
        from mla_latent_kv_29_b200 import inputs as I

        line["workloads"] = {n: workload_summary(n, args, device, peaks, flush)
                             for n in I.WORKLOADS if n not in (w.name, "tiny_b1_l128")}
        line["workloads"]["_note"] = ("the other configurations, each timed the same way as the headline "
                                      "(median of 10 steps); tiny_b1_l128 is a correctness case only")
    if args.fp8_lines:
        line["fp8_cache"] = {n: workload_summary(n, args, device, peaks, flush, fp8=True)
                             for n in (w.name, "v3_b8_l32k", "v3_b64_l8k")}
        line["fp8_cache"]["_note"] = ("the same step on the FP8 (e4m3, per-token power-of-two scale) cache: "
                                      "attention bytes = 644 per cached token + the f16 queries; the "
                                      "roofline bound is whichever of HBM and tensor time is larger")
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, st["lengths"].tolist(), args.cpu_seconds)
    return line


def e2e_pipelined(args, step, st, pieces, offs, total, h_in0, K, device):
    """Mean ms per step of K back-to-back steps through the public calls, each
    copying its inputs in from pinned host memory and its output back, with
    two staging / output buffer sets so that a step's copies overlap its
    neighbours' compute: H2D of step k on one stream (after step k - 2 is done
    with the buffers), the step on the compute stream, D2H on a third."""
    import torch

    sets = []
    for i in range(2):
        h_in = h_in0 if i == 0 else h_in0.clone().pin_memory()
        d_in = torch.empty(total, dtype=torch.uint8, device=device)
        views = [d_in[o:o + t_.numel() * t_.element_size()].view(t_.dtype).view(t_.shape)
                 for t_, o in zip(pieces, offs)]
        out = torch.empty_like(st["out"])
        h_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
        sets.append(dict(h_in=h_in, d_in=d_in, views=views, out=out, h_out=h_out, graph=None))
    saved = (st["new_seq"], st["new_pos"], st["out"])

    def bind(S):
        st["new_seq"], st["new_pos"], st["out"] = S["views"][3], S["views"][4], S["out"]

    def run_step(S):
        if S["graph"] is not None:
            S["graph"].replay()
        else:
            bind(S)
            step(x_new=S["views"][0], q_nope=S["views"][1], q_pe=S["views"][2])

    if args.graph:
        for S in sets:
            bind(S)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(x_new=S["views"][0], q_nope=S["views"][1], q_pe=S["views"][2])
            S["graph"] = g
        torch.cuda.synchronize(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_c = torch.cuda.current_stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for i in range(2):  # every event recorded once before its first wait
        ev_in[i].record(s_in)
        ev_c[i].record(s_c)
        ev_out[i].record(s_out)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):  # warm-up of the pipelined loop itself
        for k in range(2):
            S = sets[k]
            with torch.cuda.stream(s_in):
                S["d_in"].copy_(S["h_in"], non_blocking=True)
            s_c.wait_stream(s_in)
            run_step(S)
            with torch.cuda.stream(s_out):
                s_out.wait_stream(s_c)
                S["h_out"].copy_(S["out"], non_blocking=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    t0.record(s_c)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    for k in range(K):
        i = k % 2
        S = sets[i]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_c[i])  # step k - 2 has read this staging buffer
            S["d_in"].copy_(S["h_in"], non_blocking=True)
            ev_in[i].record(s_in)
        s_c.wait_event(ev_in[i])
        s_c.wait_event(ev_out[i])  # step k - 2's output has been copied out
        run_step(S)
        ev_c[i].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[i])
            S["h_out"].copy_(S["out"], non_blocking=True)
            ev_out[i].record(s_out)
    s_c.wait_stream(s_out)
    s_c.wait_stream(s_in)
    t1.record(s_c)
    torch.cuda.synchronize(device)
    barrier(device)
    st["new_seq"], st["new_pos"], st["out"] = saved
    for S in sets:
        S["graph"] = None
    return t0.elapsed_time(t1) / K


def profile_step(args, w):
    """One direct-launch step of the workload between cudaProfilerStart and
    cudaProfilerStop (for `ncu --profile-from-start off`), after the cache fill
    and the warm-up steps, with L2 flushed before it. Prints nothing."""
    import torch

    from mla_latent_kv_29_b200 import lib

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    lib.load()
    st = setup_gpu(w, device, 0)
    fp8 = args.cache == "fp8"
    if fp8:
        st["pool8"] = lib.cache_to_fp8(st["d"], st["pool"])
        st["pool"] = None
    step = make_step(w, st, args.kernel, overlap=args.overlap, fp8=fp8)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device).zero_()
    torch.cuda.synchronize(device)
    torch.cuda.profiler.start()
    step()
    torch.cuda.synchronize(device)
    torch.cuda.profiler.stop()
    assert lib.device_error() == 0, "device fault in the profiled step"


def profile_ops(args, w):
    """One step, one query projection and the two output projections (unfused
    and absorbed) of the workload's new tokens between cudaProfilerStart and
    cudaProfilerStop (for `ncu --profile-from-start off`), each after an L2
    flush, warm-ups outside. Prints nothing."""
    import torch

    from mla_latent_kv_29_b200 import inputs as I
    from mla_latent_kv_29_b200 import lib

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    lib.load()
    st = setup_gpu(w, device, 0)
    step = make_step(w, st, args.kernel, overlap=args.overlap)
    d = st["d"]
    G = w.batch * w.q_len
    qin = I.q_proj_inputs(d, G, HIDDEN, Q_RANK, seed=w.seed)
    qd = {k: (v.to(device) if v is not None else None) for k, v in qin.items()}
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 77)
    ops = [step, lambda: lib.q_proj(d, qd["x"], qd["w_qa"], qd["w_qb"], qd["positions"], q_gamma=qd["gamma"])]
    for k in (d.num_heads * d.v_head_dim, d.num_heads * d.kv_lora_rank):
        wt = (torch.randn(k, HIDDEN, generator=gen, device=device) * k ** -0.5).to(torch.bfloat16)
        x = torch.randn(G, k, generator=gen, device=device).to(torch.bfloat16)
        ops.append(lambda x=x, wt=wt: lib.o_proj(x, wt))
    for f in ops:
        for _ in range(args.warmup):
            f()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    torch.cuda.profiler.start()
    for f in ops:
        flush.zero_()
        f()
    torch.cuda.synchronize(device)
    torch.cuda.profiler.stop()
    assert lib.device_error() == 0, "device fault in the profiled operations"


def run_reference(args, w):
    """The oracle timed on the host cores (the reference arm). Each step times
    the fp64 oracle on one sequence and a quarter of the heads (plus that
    sequence's append rows) and scales by tokens and heads to the whole
    workload; the line states the seconds actually timed and the factor."""
    from mla_latent_kv_29_b200 import inputs as I

    rank, world, _ = dist_env()
    if rank != 0:
        return None
    lengths = I.context_lengths(w).tolist()
    H = w.dims.num_heads
    heads = list(range(0, H, 4))
    T = sum(lengths)
    per_step, timed_s, factors = [], 0.0, []
    for k in range(args.warmup + args.steps):
        b = k % w.batch
        s, tok = oracle_sample_seconds(w, lengths, [b], heads)
        if k >= args.warmup:
            f = (T / tok) * (H / len(heads))
            per_step.append(s * f)
            timed_s += s
            factors.append(f)
    v = statistics.mean(per_step) * 1e6
    sample = (f"each of the {args.steps} timed steps: the fp64 explicit oracle on 1 of {w.batch} sequences and "
              f"{len(heads)} of {H} heads plus its append rows ({timed_s:.2f} s of oracle time in all), scaled by "
              f"tokens and heads to the whole step (factor {statistics.mean(factors):.0f} on average)")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v / 1e3, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(w, T),
            "timing": {"value": "mean over the timed steps of (oracle seconds on the sample x scale factor)",
                       "timed_seconds": round(timed_s, 3), "samples": args.steps,
                       "scale_factor_mean": round(statistics.mean(factors), 1),
                       "step_spread": spread([x * 1e3 for x in per_step])},
            "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v3_b64_l1k_8k")
    ap.add_argument("--kernel", type=int, default=0, help="0 auto, 1 sm100 tensor-core, 2 CUDA-core")
    ap.add_argument("--soak", type=float, default=1.5, help="seconds of untimed steps while clocks are sampled")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--all-workloads", action=argparse.BooleanOptionalAction, default=True,
                    help="add a summary of every other configuration to the line")
    ap.add_argument("--fp8-lines", action=argparse.BooleanOptionalAction, default=True,
                    help="add the step on the FP8 cache for three configurations to the line")
    ap.add_argument("--overlap", action=argparse.BooleanOptionalAction, default=True,
                    help="run the append on a side stream beside the decode's query-side launches")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="replay each step from a captured CUDA graph")
    ap.add_argument("--profile-step", action="store_true",
                    help="run one step between profiler start/stop (for ncu --profile-from-start off) and exit")
    ap.add_argument("--cache", choices=["bf16", "fp8"], default="bf16",
                    help="with --profile-step: the cache format of the profiled step")
    ap.add_argument("--profile-ops", action="store_true",
                    help="run one step, one query projection and the two output projections between profiler "
                         "start/stop (for ncu --profile-from-start off) and exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from mla_latent_kv_29_b200 import inputs as I

    rank, world, _ = dist_env()
    w = I.WORKLOADS[args.workload]
    import dataclasses

    w = dataclasses.replace(w, seed=rank_seed(w.seed, rank))
    if args.profile_step:
        profile_step(args, w)
        return
    if args.profile_ops:
        profile_ops(args, w)
        return
    line = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
    if line is not None:
        print(json.dumps(line), flush=True)
    if args.impl == "ours" and world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
