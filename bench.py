#!/usr/bin/env python
"""Decode-step benchmark of the low-rank KV-cache library on B200.

One step = the whole hot path for one batch: lr_decode_step, i.e. lr_kv_append of
one new token per sequence (project, round/quantise, store) followed by
lr_attn_decode over the full context (query projection, split-sequence latent
attention, split merge and output projection).  The context is held fixed by truncating the appended
token after each step (host bookkeeping only).

By default every workload is measured and printed as its own JSON line, in the order
qwen4k, qwen16k, hybrid32k, qwen32k, qwen32k_postrope; the last line is the headline,
batch 16 at 32K context with int4 latents (the latency setup of TraceKV, "Perspective"
section of the ai4snews digest: Qwen2.5-VL-7B, batch 16, context 4K-32K), keys stored
after RoPE so that the scores run in rank space.  Inputs are seeded synthetic data
resident in HBM; L2 is
flushed before every timed step, outside the timed events (256 MiB written, then
read back, so the step neither finds its data in L2 nor pays the write-back of
dirty flush lines).

Multi-GPU: one process per GPU (torchrun); sequences are independent, so each
rank runs its own batch with its own seed and no collective on the data path
(weak scaling); timing is the max over ranks.

`--impl reference` times the CPU oracle (fp64 NumPy) on host cores on a bounded
sample of the same workload and prints the same JSON line with impl=reference.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attention µs/step & achieved HBM GB/s (% of peak), B=16, 4K–32K ctx"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TFLOPS_SUSTAINED = 1400.0

WORKLOADS = {
    "qwen4k": dict(desc="Qwen2.5-VL-7B layer: B=16, Hq=28, Hkv=4, d=128, T=4096, r_k=r_v=256 bf16 latents",
                   batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=256, length=4096,
                   quant_bits=0, layers=1),
    "qwen16k": dict(desc="Qwen2.5-VL-7B layer: B=16, Hq=28, Hkv=4, d=128, T=16384, r=352 int4 g32 latents",
                    batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=352, length=16384,
                    quant_bits=4, layers=1),
    "qwen32k": dict(desc="28 Qwen2.5-VL-7B layers: B=16, Hq=28, Hkv=4, d=128, T=32768, int4 g32 latents, "
                         "seeded per-layer ranks in [128, 448] (mean 256), keys stored before RoPE "
                         "(rebuilt and rotated per tile, theta=1e6)",
                    batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=256, length=32768,
                    quant_bits=4, layers=28, rope=True),
    "qwen32k_postrope": dict(desc="28 Qwen2.5-VL-7B layers: B=16, Hq=28, Hkv=4, d=128, T=32768, int4 g32 "
                                  "latents, seeded per-layer ranks in [128, 448] (mean 256), keys stored "
                                  "after RoPE (scores in rank space)",
                             batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=256, length=32768,
                             quant_bits=4, layers=28, rope=False),
    "qwen4k_perhead": dict(desc="Qwen2.5-VL-7B layer with one latent per KV head: B=16, Hq=28, Hkv=4, d=128, "
                                "T=4096, 4 groups of r=64 bf16 latents (the same 512 B of latents per token "
                                "as qwen4k)",
                           batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=64, length=4096,
                           quant_bits=0, layers=1, groups=4),
    "hybrid32k": dict(desc="Qwen3-8B-shaped iS-KV hybrid layer: B=8, Hq=32, Hkv=8, d=128, 32640 history "
                           "tokens of r=256 bf16 latents + an exact bf16 window of 128; every step appends "
                           "one token (the oldest window token is folded into history) and decodes; "
                           "lr_basis_sync every 128 steps, amortised into the step",
                      batch=8, n_q_heads=32, n_kv_heads=8, head_dim=128, rank=256, length=32768,
                      quant_bits=0, layers=1, window=128, sync_every=128),
}


# The default run measures every workload, one JSON line each; the last line is the
# headline: batch 16 at 32K with the keys stored after RoPE (scores in rank space), the
# HBM-bound case of the 32K configuration.
ORDER = ["qwen4k", "qwen4k_perhead", "qwen16k", "hybrid32k", "qwen32k", "qwen32k_postrope"]


def layer_ranks(workload: str, seed: int = 0):
    """(r_k, r_v) of every layer of a workload (the stored rank: groups x the group rank)."""
    import synth
    W = WORKLOADS[workload]
    if W["layers"] == 1:
        g = W.get("groups", 1)
        return [(g * W["rank"], g * W["rank"])]
    return synth.qwen32k_ranks(seed, W["layers"])


def latent_bytes_per_token(rank: int, quant_bits: int) -> int:
    if quant_bits == 4:
        g = (rank + 31) // 32
        return g * 16 + g * 4
    return rank * 2


def r_full_A(B_full, r):
    """A = r B^T of a block-diagonal basis (the generator's A for every group)."""
    return r * B_full.T


def workload_bytes(workload: str, layers: int = 0) -> int:
    """Latent (and exact-window) bytes one step reads, summed over the workload's layers
    (the first `layers` of them when given)."""
    W = WORKLOADS[workload]
    Bsz, T, qb = W["batch"], W["length"], W["quant_bits"]
    D = W["n_kv_heads"] * W["head_dim"]
    win = W.get("window", 0)
    total = 0
    ranks = layer_ranks(workload)
    for rk, rv in (ranks[:layers] if layers else ranks):
        per_tok = latent_bytes_per_token(rk, qb) + latent_bytes_per_token(rv, qb)
        total += Bsz * ((T - win) * per_tok + win * 2 * D * 2) if win else Bsz * T * per_tok
    return total


def static_config(workload: str, world: int, layers: int = 0) -> dict:
    """The `config` object of a bench line: the workload alone, identical for both arms."""
    W = WORKLOADS[workload]
    ranks = layer_ranks(workload)
    if layers:
        ranks = ranks[:layers]
    return {"workload": W["desc"], "name": workload, "batch": W["batch"], "context": W["length"],
            "layers": len(ranks),
            "ranks": sorted({r for rr in ranks for r in rr}) if len(ranks) > 1 else ranks[0][0],
            "quant_bits": W["quant_bits"], "latent_bytes_per_step": workload_bytes(workload, layers),
            "step": "lr_decode_step (= lr_kv_append + lr_attn_decode) per layer",
            "l2": "flushed before every timed step outside the events (256 MiB written, then read back "
                  "so L2 holds clean unrelated lines)",
            "parallelism": f"dp{world} (independent sequences per GPU)"}


# ----------------------------------------------------------------------------
# environment helpers
# ----------------------------------------------------------------------------


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over all ranks (identity with one process).
    Multi-GPU numbers are the slowest rank's, never a wall clock."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def percentile(values, q: float) -> float:
    """The q-th percentile (linear interpolation between order statistics)."""
    v = sorted(values)
    if not v:
        return float("nan")
    x = (len(v) - 1) * q / 100.0
    i = int(x)
    j = min(i + 1, len(v) - 1)
    return v[i] + (v[j] - v[i]) * (x - i)


def job_rate(bytes_per_step_per_rank: float, steps: int, world: int, total_ms: float) -> float:
    """Whole-job GB/s: the latent bytes every rank processed over the slowest rank's time."""
    return bytes_per_step_per_rank * steps * world / (total_ms * 1e-3) / 1e9


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU is busy."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and (not self.uuid or self.uuid in parts[0]):
                self.rows.append(parts)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def roofline_entry(kname: str, bytes_per_step: float, flops_per_step: float, kern_ms: float,
                   peaks: dict, peak_src: str, traf) -> dict:
    """The `roofline` object of the bench line for the main decode kernel (summed over the
    step's layers, `kern_ms` per step).  HBM-bound kernels: latent bytes against the measured
    copy rate.  With `flops_per_step` > 0 (keys rebuilt per tile on the tensor cores) the
    bound is the contraction, against the sustained bf16 rate (fp16 operands run at the same
    nominal rate), with the HBM view alongside."""
    gbs = bytes_per_step / (kern_ms * 1e-3) / 1e9
    timing = "CUDA events around each layer's decode kernel (separate graph capture), summed over layers"
    traffic = traf["bytes_per_launch"] if traf else None
    if flops_per_step <= 0:
        peak = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
        return {"bound": "hbm", "kernel": kname, "achieved": round(gbs, 1), "peak": peak,
                "peak_source": peak_src, "unit": "GB/s", "frac": round(gbs / peak, 4),
                "kernel_us": round(1000 * kern_ms, 2), "kernel_timing": timing, "traffic": traffic}
    tflops = flops_per_step / (kern_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_TFLOPS_SUSTAINED)
    return {"bound": "tensor", "kernel": kname, "achieved": round(tflops, 1), "peak": peak,
            "peak_source": peak_src + " (bf16 sustained; fp16 operands run at the same rate)",
            "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "flops_per_step": flops_per_step,
            "hbm_gbs": round(gbs, 1), "kernel_us": round(1000 * kern_ms, 2), "kernel_timing": timing,
            "traffic": traffic}


def basis_update_timing(L, Bsz, Hq, Hkv, d, n, dev) -> dict:
    """Median time of lr_basis_update (keys side) for one block of n rows, on a bf16 cache
    of the workload's shape whose basis rows are orthonormal (seeded)."""
    import numpy as np
    import torch
    import statistics
    import rank_kv_cache_lr_b200 as lr
    import synth
    r, D = L["rk"], Hkv * d
    rng = synth.rng_for("basis_update", "B", 0)
    B = synth.haar_orthonormal(rng, r, D)
    to = lambda x: torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(dev)
    desc = lr.make_desc(1, Hq, Hkv, d, r, r, n + 8)
    c = lr.lr_cache_create(desc, to(B.T), to(B), to(B.T), to(B))
    blk = to(rng.standard_normal((n, D)) * 0.05)
    g0 = torch.from_numpy(np.diag(synth.spectrum(r, 0.7) ** 2 * 1000.0).astype(np.float32)).to(dev)
    R = torch.empty((r, r), dtype=torch.float32, device=dev)
    Bn = torch.empty((r, D), dtype=torch.bfloat16, device=dev)
    times = []
    for i in range(4):
        g = g0.clone()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lr.lr_basis_update(c, 0, blk, g, R, Bn)
        e1.record()
        torch.cuda.synchronize()
        if i:
            times.append(e0.elapsed_time(e1))
    lr.lr_cache_destroy(c)
    return {"us_per_call": round(1000 * statistics.median(times), 1), "rank": r, "D": D, "block_rows": n,
            "timing": "CUDA events around the call, median of 3 after one warm-up"}


def paged_timing(L, p, W, dev, flush_l2) -> dict:
    """The decode kernel on the same layer held in a paged cache (128-token pages, a seeded
    random permutation of the pool as block table) beside the contiguous cache: CUDA events
    around the kernel, lr_attn_decode, L2 flushed before each call, median of 10 after 3."""
    import numpy as np
    import torch
    import statistics
    import rank_kv_cache_lr_b200 as lr
    Bsz, Hq, Hkv, d, T = W["batch"], W["n_q_heads"], W["n_kv_heads"], W["head_dim"], W["length"]
    to_dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
    desc = lr.make_desc(Bsz, Hq, Hkv, d, L["rk"], L["rv"], T, quant_bits=W["quant_bits"], dtype=lr.LR_BF16,
                        page_tokens=128)
    c = lr.lr_cache_create(desc, to_dev(p.A_k), to_dev(p.B_k), to_dev(p.A_v), to_dev(p.B_v))
    pps = T // 128
    table = np.random.default_rng(12345).permutation(Bsz * pps).astype(np.int32).reshape(Bsz, pps)
    lr.lr_cache_set_block_table(c, table)
    for s0 in range(0, p.hist_len, 1024):
        e0 = min(p.hist_len, s0 + 1024)
        lr.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k[:, s0:e0])).to(dev),
                               torch.from_numpy(np.ascontiguousarray(p.z_v[:, s0:e0])).to(dev))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(); ev1.record()
    res = {}
    for name, cache in (("paged", c), ("contiguous", L["cache"])):
        ts = []
        for i in range(13):
            flush_l2()
            lr.lr_cache_set_kernel_events(cache, ev0, ev1)
            lr.lr_attn_decode(cache, L["q"], L["out"], L["lse"])
            lr.lr_cache_set_kernel_events(cache)
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(ev0.elapsed_time(ev1))
        res[name] = statistics.median(ts)
    lr.lr_cache_destroy(c)
    return {"decode_kernel_us": round(1000 * res["paged"], 2),
            "contiguous_decode_kernel_us": round(1000 * res["contiguous"], 2),
            "table": f"random permutation of the {Bsz * pps} pages of 128 tokens",
            "timing": "CUDA events around the decode kernel of lr_attn_decode, L2 flushed before each, "
                      "median of 10 after 3"}


def prefill_timing(L, p, W, dev, flush_l2, peaks) -> dict:
    """lr_kv_prefill of the workload's whole context (B sequences x T tokens of exact keys and
    values) into an empty cache of the layer's shape: CUDA events around the call, L2 flushed
    before each, median of 5 after 2.  Bytes: the keys and values read plus the latents
    written; flops: 2 D r per token and side."""
    import numpy as np
    import torch
    import statistics
    import rank_kv_cache_lr_b200 as lr
    Bsz, Hq, Hkv, d, T = W["batch"], W["n_q_heads"], W["n_kv_heads"], W["head_dim"], W["length"]
    D, qb = Hkv * d, W["quant_bits"]
    to_dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
    desc = lr.make_desc(Bsz, Hq, Hkv, d, L["rk"], L["rv"], T, quant_bits=qb, dtype=lr.LR_BF16)
    c = lr.lr_cache_create(desc, to_dev(p.A_k), to_dev(p.B_k), to_dev(p.A_v), to_dev(p.B_v))
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    kx = (torch.randn((Bsz, T, D), generator=g, device=dev) * 0.05).to(torch.bfloat16)
    vx = (torch.randn((Bsz, T, D), generator=g, device=dev) * 0.05).to(torch.bfloat16)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for i in range(7):
        lr.lr_cache_truncate(c, 0)
        flush_l2()
        ev0.record()
        lr.lr_kv_prefill(c, kx, vx)
        ev1.record()
        torch.cuda.synchronize()
        if i >= 2:
            ts.append(ev0.elapsed_time(ev1))
    lr.lr_cache_destroy(c)
    ms = statistics.median(ts)
    nbytes = 2 * Bsz * T * D * 2 + Bsz * T * (latent_bytes_per_token(L["rk"], qb) + latent_bytes_per_token(L["rv"], qb))
    flops = 2.0 * Bsz * T * D * (L["rk"] + L["rv"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    return {"tokens": Bsz * T, "us_per_call": round(1000 * ms, 1), "GBps": round(gbs, 1),
            "TFLOPs": round(tfs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 3),
            "timing": "CUDA events around lr_kv_prefill of B x T tokens into an empty cache, L2 flushed before "
                      "each, median of 5 after 2; bytes = keys and values read + latents written"}


def traffic_record(kernel: str):
    """DRAM traffic per launch from a committed ncu summary, valid only while the kernel
    source is unchanged (matched by hash)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel]
    except (OSError, ValueError, KeyError):
        return None
    src = os.path.join(ROOT, rec["source"])
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return rec if h == rec.get("source_sha") else None


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------


def run_ours(args):
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    for wl in workloads_of(args):
        run_workload(args, wl)
        torch.cuda.empty_cache()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def workloads_of(args):
    return ORDER if args.workload == "all" else [args.workload]


def run_workload(args, workload):
    import numpy as np
    import torch

    import rank_kv_cache_lr_b200 as lr
    import synth

    rank, world, local = dist_env()
    W = WORKLOADS[workload]
    Bsz, Hq, Hkv, d, T = W["batch"], W["n_q_heads"], W["n_kv_heads"], W["head_dim"], W["length"]
    qb = W["quant_bits"]
    D = Hkv * d
    dev = torch.device("cuda", local)

    def to_dev(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)

    # seeded synthetic layers, one seed per rank (independent sequences).  Single-layer
    # workloads take their latents from the host generator; the 28-layer one draws them
    # on the device (same law: N(0,1) x i^-0.7 per rank coordinate) and quantises them
    # through lr_kv_append_latent.
    layers = []
    host_p = None
    win = W.get("window", 0)
    ranks = layer_ranks(workload)
    if args.layers:
        ranks = ranks[:args.layers]
    # The step's inputs (q, k, v of every layer) and results (out, lse of every layer) live in
    # one device buffer each, so the end-to-end run moves them with one host-to-device and one
    # device-to-host copy per step; every piece starts on a 16-byte boundary.
    D = Hkv * d
    in_bytes = (2 * Bsz * Hq * d + 2 * 2 * Bsz * D)
    out_bytes = (2 * Bsz * Hq * d + 4 * Bsz * Hq)
    assert in_bytes % 16 == 0 and out_bytes % 16 == 0 and (2 * Bsz * Hq * d) % 16 == 0 and (2 * Bsz * D) % 16 == 0
    dev_in = torch.empty(len(ranks) * in_bytes, dtype=torch.uint8, device=dev)
    dev_out = torch.empty(len(ranks) * out_bytes, dtype=torch.uint8, device=dev)

    def piece(buf, off, nbytes, dtype, shape):
        return buf[off:off + nbytes].view(dtype).view(shape)
    for li, (rk, rv) in enumerate(ranks):
        hist = T - 1
        if win:
            hist = T - win
            p = synth.make_hybrid(seed=rank, batch=Bsz, hist_len=hist, window=win, rank=rk,
                                  n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d)
            host_p = p
        elif W["layers"] == 1:
            p = synth.make_qwen(workload, seed=rank, batch=Bsz, length=hist, rank=rk, quant_bits=qb)
            host_p = p
            if W.get("groups"):   # per-group bases; the latents keep the layout [g r] per token
                g = W["groups"]
                Ak_c, Bk_c, Av_c, Bv_c, Bk_f, Bv_f = synth.grouped_bases(workload, rank, g, W["rank"], D)
                p = dataclasses.replace(p, A_k=Ak_c, B_k=Bk_c, A_v=Av_c, B_v=Bv_c)
                host_p = dataclasses.replace(p, A_k=synth.bf16_bits(r_full_A(Bk_f, W["rank"])),
                                             B_k=synth.bf16_bits(Bk_f),
                                             A_v=synth.bf16_bits(r_full_A(Bv_f, W["rank"])),
                                             B_v=synth.bf16_bits(Bv_f))
        else:
            p = synth.make_qwen(workload, seed=rank, batch=Bsz, length=0, rank=rk, rank_v=rv,
                                quant_bits=qb, layer=li)
        g = W.get("groups", 1)
        desc = lr.make_desc(Bsz, Hq, Hkv, d, rk // g, rv // g, T + (8 if win else 0), window=win, quant_bits=qb,
                            dtype=lr.LR_BF16, rope_in_kernel=1 if W.get("rope") else 0, latent_groups=g)
        cache = lr.lr_cache_create(desc, to_dev(p.A_k), to_dev(p.B_k), to_dev(p.A_v), to_dev(p.B_v))
        chunk = 1024 if W["layers"] == 1 else 2048
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000003 * (rank + 1) + li)
        sig_k = torch.arange(1, rk + 1, device=dev, dtype=torch.float32).pow(-0.7)
        sig_v = torch.arange(1, rv + 1, device=dev, dtype=torch.float32).pow(-0.7)
        for s0 in range(0, hist, chunk):
            e0 = min(hist, s0 + chunk)
            if W["layers"] == 1 or win:
                zk = torch.from_numpy(np.ascontiguousarray(p.z_k[:, s0:e0])).to(dev)
                zv = torch.from_numpy(np.ascontiguousarray(p.z_v[:, s0:e0])).to(dev)
            else:
                zk = torch.randn((Bsz, e0 - s0, rk), generator=gen, device=dev) * sig_k
                zv = torch.randn((Bsz, e0 - s0, rv), generator=gen, device=dev) * sig_v
            lr.lr_kv_append_latent(cache, zk, zv)
        for t in range(p.win_len if win else 0):   # the exact window, through lr_kv_append
            lr.lr_kv_append(cache, to_dev(np.ascontiguousarray(p.win_k[:, t])), to_dev(np.ascontiguousarray(p.win_v[:, t])))
        hp = host_p if (host_p is not None and W.get("groups")) else p
        kx, vx = synth.hybrid_token(workload, rank * 1000 + li, T - 1, Bsz, D,
                                    synth.bf16_to_f64(hp.B_k), synth.bf16_to_f64(hp.B_v), noise=1e-2 if win else 0.0)
        L = dict(cache=cache, rk=rk, rv=rv, k_h=synth.bf16_bits(kx), v_h=synth.bf16_bits(vx), q_h=p.q,
                 len0=lr.lr_cache_get_len(cache)[0])
        o_in, o_out, qb_, kb_ = li * in_bytes, li * out_bytes, 2 * Bsz * Hq * d, 2 * Bsz * D
        L["q"] = piece(dev_in, o_in, qb_, torch.bfloat16, (Bsz, Hq, d))
        L["k"] = piece(dev_in, o_in + qb_, kb_, torch.bfloat16, (Bsz, D))
        L["v"] = piece(dev_in, o_in + qb_ + kb_, kb_, torch.bfloat16, (Bsz, D))
        L["q"].copy_(to_dev(L["q_h"]))
        L["k"].copy_(to_dev(L["k_h"]))
        L["v"].copy_(to_dev(L["v_h"]))
        L["out"] = piece(dev_out, o_out, qb_, torch.bfloat16, (Bsz, Hq, d))
        L["lse"] = piece(dev_out, o_out + qb_, 4 * Bsz * Hq, torch.float32, (Bsz, Hq))
        if win:   # history latents plus the exact window tokens the step reads
            L["bytes"] = Bsz * ((T - win) * (latent_bytes_per_token(rk, qb) + latent_bytes_per_token(rv, qb))
                                + win * 2 * D * 2)
        else:
            L["bytes"] = Bsz * T * (latent_bytes_per_token(rk, qb) + latent_bytes_per_token(rv, qb))
        layers.append(L)
    torch.cuda.synchronize()
    bytes_per_step = sum(L["bytes"] for L in layers)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        # write a buffer twice the size of L2, then read it back: L2 ends up holding
        # clean unrelated lines, so the timed step neither hits its own data in L2 nor
        # pays for write-backs of the flush
        flush.zero_()
        torch.sum(flush.view(torch.int64), dim=0, out=flush_sink)
    plan = lr.lr_cache_plan(layers[0]["cache"])

    def step():
        for L in layers:   # lr_kv_append + lr_attn_decode per layer (fused launches)
            lr.lr_decode_step(L["cache"], L["k"], L["v"], L["q"], L["out"], L["lse"])
            lr.lr_cache_truncate(L["cache"], L["len0"])   # windowed caches: undo of the last append

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    # Two captures of the same step: `plain` (no event nodes, so consecutive kernels keep
    # their programmatic-dependent-launch overlap) is timed for the headline value;
    # `kev` records events around every layer's main decode kernel for the roofline.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
    for a0, a1 in kev:
        a0.record(); a1.record()
    torch.cuda.synchronize()
    n0 = lr.lr_launch_count()
    if args.graph:
        g_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_plain):
            step()
        torch.cuda.synchronize()
        launches_per_step = lr.lr_launch_count() - n0
        for L, (a0, a1) in zip(layers, kev):
            lr.lr_cache_set_kernel_events(L["cache"], a0, a1)
        g_kev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_kev):
            step()
        torch.cuda.synchronize()
        for L in layers:
            lr.lr_cache_set_kernel_events(L["cache"])
        run, run_kev = g_plain.replay, g_kev.replay
    else:
        step()
        torch.cuda.synchronize()
        launches_per_step = lr.lr_launch_count() - n0

        def run_kev():
            for L, (a0, a1) in zip(layers, kev):
                lr.lr_cache_set_kernel_events(L["cache"], a0, a1)
            step()
            for L in layers:
                lr.lr_cache_set_kernel_events(L["cache"])
        run = step
    for _ in range(3):
        run()
        run_kev()
    torch.cuda.synchronize()

    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    sampler = ClockSampler(uuid)
    sampler.start()
    t_end = time.time() + args.load_seconds          # sustained load so the sampler sees the
    while time.time() < t_end:                        # clocks of this very step
        for _ in range(max(1, 50 // len(layers))):
            run()
        torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush_l2()
        ev[i][0].record()
        run()
        ev[i][1].record()
    torch.cuda.synchronize()
    barrier()
    launches = launches_per_step * K
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)
    # the same step with a warm L2 (no flush between steps): labelled, not the graded value
    wev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        wev[i][0].record()
        run()
        wev[i][1].record()
    torch.cuda.synchronize()
    warm_ms = [a.elapsed_time(b) for a, b in wev]
    # roofline: the main decode kernel of every layer, timed inside the `kev` capture
    kern_ms = []
    for i in range(K):
        flush_l2()
        run_kev()
        torch.cuda.synchronize()
        kern_ms.append(sum(a0.elapsed_time(a1) for a0, a1 in kev))

    # end to end with host buffers (pinned): H2D of the step's inputs, the step through
    # the public API (replayed graph of lr_kv_append + lr_attn_decode per layer), D2H of
    # the results
    host_in = torch.empty(dev_in.numel(), dtype=torch.uint8).pin_memory()
    host_out = torch.empty(dev_out.numel(), dtype=torch.uint8).pin_memory()
    host_in.copy_(dev_in.cpu())      # the step's inputs, in the device buffer's layout

    def run_e2e_eager():
        dev_in.copy_(host_in, non_blocking=True)
        run()
        host_out.copy_(dev_out, non_blocking=True)
    run_e2e = run_e2e_eager
    if args.graph:
        # the copies and the step as one graph (pinned host buffers: the copies become graph
        # nodes), as a serving loop would replay it
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            dev_in.copy_(host_in, non_blocking=True)
            step()
            host_out.copy_(dev_out, non_blocking=True)
        torch.cuda.synchronize()
        run_e2e = g_e2e.replay
        for _ in range(3):
            run_e2e()
        torch.cuda.synchronize()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    barrier()
    for i in range(K):
        flush_l2()
        e2e_ev[i][0].record()
        run_e2e()
        e2e_ev[i][1].record()
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)
    h2d = host_in.numel()
    d2h = host_out.numel()

    # basis sync (windowed workloads): seeded Haar rotations, B' = R^T B, A' = A R, timed
    # alone; its cost is amortised over `sync_every` steps in the headline value
    sync = None
    if W.get("sync_every"):
        L = layers[0]
        Rk = synth.sync_rotation(rank, 0, L["rk"], "k")
        Rv = synth.sync_rotation(rank, 0, L["rv"], "v")
        Bk0, Bv0 = synth.bf16_to_f64(host_p.B_k), synth.bf16_to_f64(host_p.B_v)
        Ak0, Av0 = synth.bf16_to_f64(host_p.A_k), synth.bf16_to_f64(host_p.A_v)
        sargs = (torch.from_numpy(Rk.astype(np.float32)).to(dev), torch.from_numpy(Rv.astype(np.float32)).to(dev),
                 to_dev(synth.bf16_bits(Rk.T @ Bk0)), to_dev(synth.bf16_bits(Rv.T @ Bv0)),
                 to_dev(synth.bf16_bits(Ak0 @ Rk)), to_dev(synth.bf16_bits(Av0 @ Rv)))
        lr.lr_basis_sync(L["cache"], *sargs)
        torch.cuda.synchronize()
        sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
        for a0, a1 in sev:
            flush_l2()
            a0.record()
            lr.lr_basis_sync(L["cache"], *sargs)
            a1.record()
        torch.cuda.synchronize()
        sync_ms = statistics.median(a0.elapsed_time(a1) for a0, a1 in sev)
        sync_bytes = 2 * 2 * Bsz * (T - W["window"]) * L["rk"] * 2      # K and V history, read + write
        sync = {"us_per_call": round(1000 * sync_ms, 2), "every_steps": W["sync_every"],
                "us_per_step_amortised": round(1000 * sync_ms / W["sync_every"], 3),
                "GBps": round(sync_bytes / (sync_ms * 1e-3) / 1e9, 1)}
        total_ms += K * sync_ms / W["sync_every"]
        e2e_ms += K * sync_ms / W["sync_every"]
        # the basis update that produces R and the new basis from a folded block of
        # `sync_every` exact key rows (lr_basis_update, fp64 on the GPU), timed on a cache of
        # the same shape with an orthonormal basis; reported beside the decode, not in it
        upd = basis_update_timing(L, Bsz, Hq, Hkv, d, W["sync_every"], dev)
        upd["every_steps"] = W["sync_every"]
        upd["us_per_step_amortised"] = round(upd["us_per_call"] / W["sync_every"], 2)
        sync["basis_update"] = upd

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    value = job_rate(bytes_per_step, K, world, total_ms)
    peaks, peak_src = measured_peaks()
    kern_mean = statistics.mean(kern_ms)
    kname = ("decode_tc_i4" if qb == 4 else "decode_tc") if plan.path == lr.LR_PATH_TC else "decode_simt"
    rope = bool(W.get("rope"))
    if rope:
        kname += "_rope"
    traf = traffic_record(f"{kname}:{workload}")
    # Keys stored before RoPE are rebuilt per tile on the tensor cores: the contraction
    # (2 r_k D per token for the keys, 2 r_v Hq for the value mix) bounds that kernel, not
    # HBM; fp16 operands run at the bf16 rate, and the kernel runs inside a long step
    # (sustained peak).
    roof_flops = sum(Bsz * T * (2 * L["rk"] * D + 2 * L["rv"] * Hq) for L in layers) if rope else 0.0
    assert bytes_per_step == workload_bytes(workload, len(layers))
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "us_per_step": round(1000 * total_ms / K, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4+bf16" if qb else "bf16",
        "data": "synthetic (seeded; one seed per rank)",
        "config": static_config(workload, world, args.layers),
        "run": {"decode_path": "tcgen05" if plan.path == lr.LR_PATH_TC else "simt",
                "splits": plan.n_splits, "cuda_graph": bool(args.graph),
                "launches_per_step": launches_per_step,
                "step_us": {"median": round(1000 * statistics.median(step_ms), 2),
                            "p10": round(1000 * percentile(step_ms, 10), 2),
                            "p90": round(1000 * percentile(step_ms, 90), 2),
                            "of": "this rank's timed steps, L2 flushed before each"},
                "warm_l2_step_us": {"median": round(1000 * statistics.median(warm_ms), 2),
                                    "note": "the same step replayed back to back without the L2 flush "
                                            "(latents partly or wholly L2-resident); not the graded value"}},
        "roofline": roofline_entry(kname, bytes_per_step, roof_flops, kern_mean, peaks, peak_src, traf),
        "e2e": {"value": round(job_rate(bytes_per_step, K, world, e2e_ms), 2), "unit": "GB/s",
                "us_per_step": round(1000 * e2e_ms / K, 2), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "pinned host inputs -> lr_decode_step per layer -> pinned host outputs"
                        + (", replayed as one CUDA graph" if args.graph else "")},
        "gpu_launches": launches,
        "clocks": sampler.summary(),
    }
    if sync is not None:
        res["run"]["basis_sync"] = sync
    if W["layers"] == 1 and not win and not W.get("groups") and world == 1:
        # the same layer in a paged cache: paging moves no bytes and adds no work
        res["run"]["paged"] = paged_timing(layers[0], host_p, W, dev, flush_l2)
        # bulk prefill of the layer's whole context (the cache fill from exact keys / values)
        res["run"]["prefill"] = prefill_timing(layers[0], host_p, W, dev, flush_l2, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(workload, host_p, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(res), flush=True)
    run = run_kev = run_e2e = None
    if args.graph:
        del g_plain, g_kev, g_e2e
    for L in layers:
        lr.lr_cache_destroy(L["cache"])


# ----------------------------------------------------------------------------
# the CPU oracle as baseline / reference arm
# ----------------------------------------------------------------------------


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step_sample(p, rows, seconds):
    """Time the oracle's decode over `rows` batch rows (all heads) of problem p, repeated
    for about `seconds`; returns (bytes of latents processed per second, s per row-step)."""
    import numpy as np
    from oracle import attention, quant
    t0 = time.time()
    done = 0
    nbytes = 0
    per_tok = latent_bytes_per_token(p.rank_k, p.quant_bits)
    while True:
        for b in rows:
            if p.quant_bits == 4:
                c, s, z = quant.quantize_int4(p.z_k[b]); zk = quant.dequantize_int4(c, s, z, p.rank_k)
                c, s, z = quant.quantize_int4(p.z_v[b]); zv = quant.dequantize_int4(c, s, z, p.rank_v)
            elif p.dtype == "bf16":
                zk = quant.round_to_bf16(p.z_k[b]); zv = quant.round_to_bf16(p.z_v[b])
            else:
                zk = np.asarray(p.z_k[b], np.float64); zv = np.asarray(p.z_v[b], np.float64)
            qv = p.to_f64(p.q[b:b + 1])
            Bk, Bv = p.to_f64(p.B_k), p.to_f64(p.B_v)
            wk = wv = None
            if p.win_k is not None and p.win_len:
                wk, wv = p.to_f64(p.win_k[b:b + 1]), p.to_f64(p.win_v[b:b + 1])
            attention.decode(qv, zk[None], zv[None], Bk, Bv, p.n_kv_heads, None,
                             p.rope_theta if p.rope else None, wk, wv)
            done += 1
            nbytes += p.hist_len * 2 * per_tok + (p.win_len * 2 * p.kv_dim * 2 if wk is not None else 0)
        el = time.time() - t0
        if el >= seconds:
            return nbytes / el, el / done, done


def host_problem(workload, seed, batch):
    """A host-side instance of (the first layer of) a workload for the CPU oracle."""
    import synth
    W = WORKLOADS[workload]
    if W.get("window"):
        return synth.make_hybrid(seed=seed, batch=batch, hist_len=W["length"] - W["window"], window=W["window"],
                                 rank=W["rank"], n_q_heads=W["n_q_heads"], n_kv_heads=W["n_kv_heads"],
                                 head_dim=W["head_dim"])
    if W["layers"] == 1:
        g = W.get("groups", 1)
        p = synth.make_qwen(workload, seed=seed, batch=batch, length=W["length"] - 1, rank=g * W["rank"],
                            quant_bits=W["quant_bits"])
        if g > 1:   # the block-diagonal bases of the per-group ones
            D = W["n_kv_heads"] * W["head_dim"]
            *_, Bk_f, Bv_f = synth.grouped_bases(workload, seed, g, W["rank"], D)
            p = dataclasses.replace(p, A_k=synth.bf16_bits(r_full_A(Bk_f, W["rank"])), B_k=synth.bf16_bits(Bk_f),
                                    A_v=synth.bf16_bits(r_full_A(Bv_f, W["rank"])), B_v=synth.bf16_bits(Bv_f))
        return p
    return synth.make_qwen32k_layer(0, seed=seed, batch=batch, length=W["length"] - 1, rope=bool(W.get("rope")))


def single_core_timings(seconds):
    """The oracle on one host core for the two small configurations (the tiny fp32 case
    and the 4K bf16 layer): one batch row, all heads; bounded to `seconds` in total."""
    import synth
    from threadpoolctl import threadpool_limits
    out = {}
    with threadpool_limits(limits=1):
        for name, p in (("tiny", synth.make_tiny()), ("qwen4k", host_problem("qwen4k", 0, 1))):
            bps, s_per_row, n = oracle_step_sample(p, [0], seconds / 2)
            out[name] = {"GBps": round(bps / 1e9, 5), "ms_per_row": round(1e3 * s_per_row, 3), "rows": n,
                         "cores": 1}
    return out


def cpu_baseline(workload, p, seconds):
    if p is None:
        p = host_problem(workload, 0, 1)
    bps, s_per_row, n = oracle_step_sample(p, [0], seconds)
    res = {"value": round(bps / 1e9, 4), "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
           "us_per_step_equiv": round(1e6 * s_per_row * p.batch, 1),
           "sample": f"{n} oracle decodes of batch row 0 (all {p.n_q_heads} heads, T={p.hist_len}) of the "
                     f"{workload} step (first layer), fp64 NumPy; GB/s of latents processed"}
    if workload == "qwen4k":
        res["single_core"] = single_core_timings(min(seconds, 8.0))
    return res


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    for wl in workloads_of(args):
        run_reference_workload(args, wl, world)


def run_reference_workload(args, workload, world):
    W = WORKLOADS[workload]
    p = host_problem(workload, 0, 1)
    for _ in range(args.warmup):
        oracle_step_sample(p, [0], 0.0)
    t0 = time.time()
    per = max(0.5, args.cpu_seconds / max(args.steps, 1))
    tot_bytes = 0.0
    for _ in range(args.steps):
        bps, _, n = oracle_step_sample(p, [0], per)
        tot_bytes += bps * per
    el = time.time() - t0
    value = tot_bytes / el / 1e9
    cores = _blas_threads()
    us_step = 1e6 * el / args.steps
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(us_step / 1000, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": static_config(workload, world, args.layers),
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                            "sample": "each step: repeated oracle decodes of batch row 0 (all heads) for a "
                                      f"bounded {per:.1f} s; value = latent bytes processed per second"},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(WORKLOADS),
                    help="one workload, or all of them (one line each, the 32K rank-space headline last)")
    ap.add_argument("--layers", type=int, default=0,
                    help="only the first N layers of a multi-layer workload (profiling runs; 0 = all)")
    ap.add_argument("--load-seconds", type=float, default=1.5)
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the step's calls directly instead of replaying a CUDA graph")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
