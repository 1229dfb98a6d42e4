#!/usr/bin/env python
"""Decode-step benchmark of the low-rank KV-cache library on B200.

One step = the whole hot path for one batch: lr_decode_step, i.e. lr_kv_append of
one new token per sequence (project, round/quantise, store) followed by
lr_attn_decode over the full context (query projection, split-sequence latent
attention, split merge and output projection).  The context is held fixed by truncating the appended
token after each step (host bookkeeping only).

Default workload: one Qwen2.5-VL-7B-shaped layer, batch 16, 28 query heads over
4 KV heads, head_dim 128, 4096 tokens of bf16 rank-256 latents (the latency
setup of TraceKV, "Perspective" section of the ai4snews digest: batch 16,
context 4K-32K).  Inputs are seeded synthetic data resident in HBM; L2 is
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

WORKLOADS = {
    "qwen4k": dict(desc="Qwen2.5-VL-7B layer: B=16, Hq=28, Hkv=4, d=128, T=4096, r_k=r_v=256 bf16 latents",
                   batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=256, length=4096,
                   quant_bits=0),
    "qwen16k": dict(desc="Qwen2.5-VL-7B layer: B=16, Hq=28, Hkv=4, d=128, T=16384, r=352 int4 g32 latents",
                    batch=16, n_q_heads=28, n_kv_heads=4, head_dim=128, rank=352, length=16384,
                    quant_bits=4),
}


def latent_bytes_per_token(rank: int, quant_bits: int) -> int:
    if quant_bits == 4:
        g = (rank + 31) // 32
        return g * 16 + g * 4
    return rank * 2


# ----------------------------------------------------------------------------
# environment helpers
# ----------------------------------------------------------------------------


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


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
    import numpy as np
    import torch

    import rank_kv_cache_lr_b200 as lr
    import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    W = WORKLOADS[args.workload]
    Bsz, Hq, Hkv, d, r, T = W["batch"], W["n_q_heads"], W["n_kv_heads"], W["head_dim"], W["rank"], W["length"]
    qb = W["quant_bits"]
    D = Hkv * d

    # seeded synthetic layer, one seed per rank (independent sequences)
    p = synth.make_qwen(args.workload, seed=rank, batch=Bsz, length=T - 1, rank=r, quant_bits=qb)
    dev = torch.device("cuda", local)

    def to_dev(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)

    desc = lr.make_desc(Bsz, Hq, Hkv, d, r, r, T, quant_bits=qb, dtype=lr.LR_BF16)
    cache = lr.lr_cache_create(desc, to_dev(p.A_k), to_dev(p.B_k), to_dev(p.A_v), to_dev(p.B_v))
    chunk = 1024
    for s in range(0, T - 1, chunk):
        e = min(T - 1, s + chunk)
        lr.lr_kv_append_latent(cache, torch.from_numpy(np.ascontiguousarray(p.z_k[:, s:e])).to(dev),
                               torch.from_numpy(np.ascontiguousarray(p.z_v[:, s:e])).to(dev))
    kx, vx = synth.hybrid_token(args.workload, rank, T - 1, Bsz, D,
                                synth.bf16_to_f64(p.B_k), synth.bf16_to_f64(p.B_v))
    k_h, v_h = synth.bf16_bits(kx), synth.bf16_bits(vx)
    k_d, v_d, q_d = to_dev(k_h), to_dev(v_h), to_dev(p.q)
    out = torch.empty_like(q_d)
    lse = torch.empty((Bsz, Hq), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        # write a buffer twice the size of L2, then read it back: L2 ends up holding
        # clean unrelated lines, so the timed step neither hits its own data in L2 nor
        # pays for write-backs of the flush
        flush.zero_()
        torch.sum(flush.view(torch.int64), dim=0, out=flush_sink)
    plan = lr.lr_cache_plan(cache)

    def step(kk, vv, qq, oo, ll):
        lr.lr_decode_step(cache, kk, vv, qq, oo, ll)   # lr_kv_append + lr_attn_decode, fused launches
        lr.lr_cache_truncate(cache, T - 1)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        flush_l2()
        step(k_d, v_d, q_d, out, lse)
    torch.cuda.synchronize()

    # kernel-only events around the main decode kernel (recorded by the library)
    kev0, kev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kev0.record(); kev1.record()
    torch.cuda.synchronize()
    lr.lr_cache_set_kernel_events(cache, kev0, kev1)
    graph = None
    n0 = lr.lr_launch_count()
    if args.graph:
        # the step is replayed as a CUDA graph: the context is fixed (append at slot T-1,
        # decode over T tokens, truncate back), so the captured launches are the step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(k_d, v_d, q_d, out, lse)
        torch.cuda.synchronize()
        run = graph.replay
    else:
        step(k_d, v_d, q_d, out, lse)
        torch.cuda.synchronize()
        run = lambda: step(k_d, v_d, q_d, out, lse)  # noqa: E731
    launches_per_step = lr.lr_launch_count() - n0
    for _ in range(3):
        run()
    torch.cuda.synchronize()

    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    sampler = ClockSampler(uuid)
    sampler.start()
    t_end = time.time() + args.load_seconds          # sustained load so the sampler sees the
    while time.time() < t_end:                        # clocks of this very step
        for _ in range(50):
            run()
        torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    kern_ms = []
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush_l2()
        ev[i][0].record()
        run()
        ev[i][1].record()
        kev1.synchronize()
        kern_ms.append(kev0.elapsed_time(kev1))
    torch.cuda.synchronize()
    barrier()
    launches = launches_per_step * K
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)

    # end to end with host buffers (pinned): H2D of the step's inputs, the step through
    # the public API (replayed graph of lr_kv_append + lr_attn_decode), D2H of the result
    q_host = torch.from_numpy(np.ascontiguousarray(p.q).view(np.int16)).view(torch.bfloat16).pin_memory()
    k_host = torch.from_numpy(k_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    v_host = torch.from_numpy(v_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((Bsz, Hq, d), dtype=torch.bfloat16).pin_memory()
    lse_host = torch.empty((Bsz, Hq), dtype=torch.float32).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    barrier()
    for i in range(K):
        flush_l2()
        e2e_ev[i][0].record()
        q_d.copy_(q_host, non_blocking=True)
        k_d.copy_(k_host, non_blocking=True)
        v_d.copy_(v_host, non_blocking=True)
        run()
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)
        e2e_ev[i][1].record()
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    lr.lr_cache_set_kernel_events(cache)
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)
    h2d = (q_host.numel() + k_host.numel() + v_host.numel()) * 2
    d2h = out_host.numel() * 2 + lse_host.numel() * 4

    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([total_ms, e2e_ms, max(kern_ms) if kern_ms else 0.0], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, e2e_ms = float(t[0]), float(t[1])

    bytes_per_step = Bsz * T * 2 * latent_bytes_per_token(r, qb)
    value = bytes_per_step * K * world / (total_ms * 1e-3) / 1e9
    peaks, peak_src = measured_peaks()
    kern_mean = statistics.mean(kern_ms)
    achieved = bytes_per_step / (kern_mean * 1e-3) / 1e9
    kname = "decode_tc" if plan.path == lr.LR_PATH_TC else "decode_simt"
    traf = traffic_record(kname)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "us_per_step": round(1000 * total_ms / K, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4+bf16" if qb else "bf16",
        "data": "synthetic (seeded; one seed per rank)",
        "config": {"workload": W["desc"], "batch": Bsz, "context": T, "rank": r,
                   "quant_bits": qb, "latent_bytes_per_step": bytes_per_step,
                   "step": "lr_decode_step (= lr_kv_append + lr_attn_decode)", "l2": "flushed before every timed step outside the events (256 MiB written, then read back so L2 holds clean unrelated lines)",
                   "parallelism": f"dp{world} (independent sequences per GPU)",
                   "decode_path": "tcgen05" if plan.path == lr.LR_PATH_TC else "simt",
                   "splits": plan.n_splits, "cuda_graph": bool(args.graph),
                   "launches_per_step": launches_per_step},
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": round(achieved, 1),
                     "peak": peaks.get("hbm_gbs", FALLBACK_HBM_GBS), "peak_source": peak_src,
                     "unit": "GB/s", "frac": round(achieved / peaks.get("hbm_gbs", FALLBACK_HBM_GBS), 4),
                     "kernel_us": round(1000 * kern_mean, 2),
                     "traffic": (traf["bytes_per_launch"] if traf else None)},
        "e2e": {"value": round(bytes_per_step * K * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "us_per_step": round(1000 * e2e_ms / K, 2), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(args.workload, p, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(res), flush=True)
    del graph
    lr.lr_cache_destroy(cache)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


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
            else:
                zk = quant.round_to_bf16(p.z_k[b]); zv = quant.round_to_bf16(p.z_v[b])
            qv = (p.q[b:b + 1].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            Bk = (p.B_k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            Bv = (p.B_v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            attention.decode(qv, zk[None], zv[None], Bk, Bv, p.n_kv_heads)
            done += 1
            nbytes += p.hist_len * 2 * per_tok
        el = time.time() - t0
        if el >= seconds:
            return nbytes / el, el / done, done


def cpu_baseline(workload, p, seconds):
    bps, s_per_row, n = oracle_step_sample(p, [0], seconds)
    return {"value": round(bps / 1e9, 4), "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
            "us_per_step_equiv": round(1e6 * s_per_row * p.batch, 1),
            "sample": f"{n} oracle decodes of batch row 0 (all {p.n_q_heads} heads, T={p.hist_len}) of the "
                      f"{workload} step, fp64 NumPy; GB/s of latents processed"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import synth
    W = WORKLOADS[args.workload]
    p = synth.make_qwen(args.workload, seed=0, batch=W["batch"], length=W["length"] - 1,
                        rank=W["rank"], quant_bits=W["quant_bits"])
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
           "config": {"workload": W["desc"], "batch": W["batch"], "context": W["length"], "rank": W["rank"]},
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
    ap.add_argument("--workload", default="qwen4k", choices=sorted(WORKLOADS))
    ap.add_argument("--load-seconds", type=float, default=1.5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
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
