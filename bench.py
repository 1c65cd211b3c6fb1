"""Benchmark of the MoBA causal-prefill forward pass on B200.

One step = one whole forward pass (pool keys, gate + top-k, routing, past-block
attention, own-block attention + online-softmax merge) over one batch of seeded
synthetic inputs already resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own independent replica of the workload
(the path has no cross-GPU exchange: problems shard by sequence and KV-head group),
so scaling is weak; the timed region is bracketed by barriers and its length is the
maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoBA fwd effective TFLOP/s & tokens/s at 1M ctx; % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w: synth.Workload) -> str:
    lens = "+".join(str(x) for x in w.seqlens)
    extra = []
    if w.rope_theta:
        extra.append("RoPE theta=%g" % w.rope_theta)
    if w.plant:
        extra.append("planted relevance %.1f" % w.plant)
    return "%s: seqs=%s Hq=%d Hkv=%d D=%d block_size=%d top_k=%d %s" % (
        w.name, lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.top_k,
        ", ".join(extra))


def flop_counts(w: synth.Workload, routed_rows: int) -> dict:
    """Algorithmic FLOPs of one pass: attention over unmasked attended keys, and the gate."""
    D, hq, bs = w.head_dim, w.num_q_heads, w.block_size
    self_keys = 0
    gate_dots = 0
    for L in w.seqlens:
        p = np.arange(L, dtype=np.int64)
        self_keys += int(np.sum(p % bs + 1))
        gate_dots += int(np.sum(p // bs))
    past = 4 * D * bs * routed_rows
    own = 4 * D * hq * self_keys
    gate = 2 * D * hq * gate_dots
    return {"past": past, "own": own, "gate": gate, "attn": past + own}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def past_kernel_traffic(routed_rows: int):
    """DRAM bytes per launch of the past-block attention kernel, from the committed ncu
    record scaled by routed rows, or None when the kernel sources changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "attn_past_traffic.json")
    if not os.path.exists(path):
        return None, "no capture"
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for name in rec["source_files"]:
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["source_sha256"]:
        return None, "kernel changed since the capture"
    per_row = (rec["dram_bytes_read"] + rec["dram_bytes_write"]) / rec["routed_rows"]
    return per_row * routed_rows, "scaled from the %s capture by routed rows" % rec["workload"]


def max_over_ranks(value: float, dist, device=None) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's time)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Units all ranks processed over the timed region, per second of its slowest rank."""
    return units_per_rank * world * steps / (max_ms / 1e3)


def make_host_inputs(w: synth.Workload, pinned: bool, nthreads: int | None = None):
    import torch
    out = {}
    for which in ("q", "k", "v"):
        shape = (w.total_tokens, w.heads(which), w.head_dim)
        t = torch.empty(shape, dtype=torch.int16, pin_memory=pinned)
        w.fill(which, out=t.numpy().view(np.uint16), nthreads=nthreads)
        out[which] = t.view(torch.bfloat16)
    return out


# --------------------------------------------------------------------------- CPU oracle
def oracle_rows_per_second(w: synth.Workload, K: np.ndarray, V: np.ndarray, budget_s: float,
                           seed: int = 0):
    """Time the fp64 oracle on a bounded, seeded sample of query rows of the workload.

    Returns (tokens/s extrapolated to the whole pass, rows timed, seconds, threads, pool s).
    The pooled keys are computed once over all of K (timed) and the per-row cost is
    extrapolated to T * Hq rows.
    """
    import oracle
    pr = oracle.Problem(w.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                        w.top_k, dtype="bf16")
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    kbar = oracle.pool_keys(pr, K, nthreads=threads)
    pool_s = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    T, hq = w.total_tokens, w.num_q_heads
    done_rows, done_s = 0, 0.0
    n = max(threads, 16)
    while done_s < budget_s and n > 0:
        tok = rng.integers(0, T, size=n)
        hd = rng.integers(0, hq, size=n)
        qrows = w.rows("q", tok, hd)
        t0 = time.perf_counter()
        oracle.rows(pr, qrows, K, V, kbar, tok, hd, nthreads=threads)
        dt = time.perf_counter() - t0
        done_rows += n
        done_s += dt
        per_row = done_s / done_rows
        n = int(min(max((budget_s - done_s) / per_row, 0), 4 * done_rows + threads))
    per_row = done_s / max(done_rows, 1)
    full_s = pool_s + per_row * T * hq
    return T / full_s, done_rows, done_s, threads, pool_s


# --------------------------------------------------------------------------- our arm
def run_ours(args, w: synth.Workload, rank: int, world: int, dist) -> dict | None:
    import torch
    import block_sparse_attention_gate_b200 as mb

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    host = make_host_inputs(w, pinned=True, nthreads=max(1, (os.cpu_count() or 1) // world))
    Q = host["q"].to(dev, non_blocking=True)
    K = host["k"].to(dev, non_blocking=True)
    V = host["v"].to(dev, non_blocking=True)
    p = mb.MobaParams(w.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                      w.top_k)
    ws = mb.alloc_workspace(p, dev)
    T, hq, D = Q.shape
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device=dev)
    sel = torch.empty((T, hq, w.top_k), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    LSE = torch.empty((T, hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    stages = ("pool", "gate", "route", "past", "own")

    def step(ev):
        ev[0].record(stream)
        mb.moba_pool_keys(p, K, kbar, stream)
        ev[1].record(stream)
        mb.moba_gate_topk(p, Q, kbar, sel, ws, stream)
        ev[2].record(stream)
        mb.moba_route(p, sel, ws, stream)
        ev[3].record(stream)
        mb.moba_attn_past(p, Q, K, V, ws, stream)
        ev[4].record(stream)
        mb.moba_attn_self_merge(p, Q, K, V, sel, ws, O, LSE, stream)
        ev[5].record(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    warm = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(args.warmup):
        step(warm)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    total_ms = evs[0][0].elapsed_time(evs[-1][5])
    stage_ms = {s: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j, s in enumerate(stages)}
    t_max = max_over_ranks(total_ms, dist, dev)
    routed = int((sel[:, :, 1:] >= 0).sum().item()) if w.top_k > 1 else 0
    # sel slot >= 1 is valid exactly when it names a past block; verify the count from the rows
    fl = flop_counts(w, routed)
    ms_step = t_max / args.steps
    tokens_per_s = job_throughput(T, world, args.steps, t_max)

    # ----- end to end through the public call with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        # the public host-buffer call: per-KV-group slices copied and computed over 3 streams
        O_host = torch.empty(O.shape, dtype=torch.bfloat16, pin_memory=True)
        L_host = torch.empty(LSE.shape, dtype=torch.float32, pin_memory=True)
        streams = [torch.cuda.Stream(dev) for _ in range(3)]
        staging = torch.empty(max(mb.moba_host_staging_size(p, len(streams)), 256), dtype=torch.uint8,
                              device=dev)
        n_e2e = max(1, min(args.steps, 3))
        main_stream = torch.cuda.current_stream(dev)

        def e2e_run(n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(main_stream)
            for s_ in streams:
                s_.wait_event(a)
            for _ in range(n):
                mb.moba_fwd_host(p, host["q"], host["k"], host["v"], O_host, L_host, staging, streams)
            for s_ in streams:
                ev = torch.cuda.Event()
                ev.record(s_)
                main_stream.wait_event(ev)
            b.record(main_stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b)

        e2e_run(1)
        if dist is not None:
            dist.barrier()
        e_ms = max_over_ranks(e2e_run(n_e2e), dist, dev)
        h2d = sum(host[x].numel() * 2 for x in ("q", "k", "v"))
        d2h = O.numel() * 2 + LSE.numel() * 4
        e2e = {"value": job_throughput(T, world, n_e2e, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e}

    traffic, traffic_note = past_kernel_traffic(routed)
    peaks, peak_kind = load_peaks()
    peak_tf = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    past_s = stage_ms["past"] / 1e3
    achieved = fl["past"] / past_s / 1e12 if past_s > 0 else 0.0
    attn_s = (stage_ms["past"] + stage_ms["own"]) / 1e3
    eff_tf = (fl["attn"] + fl["gate"]) / (ms_step / 1e3) / 1e12
    res = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded splitmix64/Box-Muller normals, RoPE, planted relevance per recipe)",
        "config": {"workload": workload_desc(w), "seq_len": w.max_seqlen, "global_batch": w.num_seqs * world,
                   "total_tokens_per_gpu": T, "parallelism": "replicas%d" % world,
                   "l2": "inputs larger than L2 (Q alone %.1f GB)" % (Q.numel() * 2 / 1e9)},
        "eff_tflops": eff_tf,
        "attn_eff_tflops": fl["attn"] / attn_s / 1e12 if attn_s > 0 else 0.0,
        "pct_bf16_peak": 100.0 * eff_tf / peak_tf,
        "stage_ms": stage_ms,
        "flops": fl,
        "routed_rows": routed,
        "roofline": {"bound": "tensor", "kernel": "past-block attention", "achieved": achieved,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                     "peak_kind": "%s bf16 sustained (kernel timed inside a long step)" % peak_kind,
                     "traffic": traffic, "traffic_note": traffic_note},
        "clocks": clk,
        "gpu_launches": mb.moba_launches_per_forward(p) * args.steps,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        Kh = host["k"].view(torch.int16).numpy().view(np.uint16)
        Vh = host["v"].view(torch.int16).numpy().view(np.uint16)
        tps, nrows, secs, thr, pool_s = oracle_rows_per_second(w, Kh, Vh, args.cpu_seconds)
        res["cpu_baseline"] = {
            "value": tps, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": "%d random query rows of the same workload in %.1f s plus one pooling pass over "
                      "all keys (%.1f s); per-row time extrapolated to all T*Hq rows" % (nrows, secs, pool_s)}
    return res


def run_reference(args, w: synth.Workload, rank: int) -> dict | None:
    """The oracle (fp64 CPU, all host cores) on a bounded sample of the same workload."""
    if rank != 0:
        return None
    Kh = w.fill("k")
    Vh = w.fill("v")
    vals, rows_all, secs_all = [], 0, 0.0
    for i in range(args.warmup + args.steps):
        tps, nrows, secs, thr, pool_s = oracle_rows_per_second(
            w, Kh, Vh, args.ref_seconds, seed=i)
        if i >= args.warmup:
            vals.append(tps)
            rows_all += nrows
            secs_all += secs
    v = statistics.mean(vals)
    T = w.total_tokens
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * T / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": workload_desc(w), "seq_len": w.max_seqlen, "global_batch": w.num_seqs},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": "%d random query rows over %d steps (%.1f s) plus pooling, "
                                   "extrapolated to all rows" % (rows_all, args.steps, secs_all)},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="prefill1m", choices=sorted(synth.CONFIGS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    args = ap.parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = synth.CONFIGS[args.config]
    if args.impl == "reference":
        res = run_reference(args, w, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
        dist = tdist
    try:
        res = run_ours(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
