"""Benchmark of the MoBA causal-prefill forward pass on B200.

One step = one whole forward pass (pool keys, gate + top-k, routing, past-block
attention, own-block attention + online-softmax merge) over one batch of seeded
synthetic inputs already resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Besides the headline workload (1M tokens by default) the line carries
  * ``configs``: the other long-context workloads (128K GQA, packed varlen) timed the
    same way, with the attention's fraction of the measured bf16 peaks;
  * ``dense_causal``: dense causal attention on the same GPU (torch SDPA, outside the
    MoBA timed region) at the headline workload and at 32K MHA, and the library's own
    full mode (top_k >= number of blocks) at 32K MHA;
  * ``prefill10m_group``: a 10M-token sequence with one KV-head group (the unit a full
    32/8-head 10M pass runs in, group by group);
  * ``backward``, ``decode``, ``mask_based``: the backward pass at the headline workload,
    gated decode over its keys and values as KV caches (with dense decode beside it), and
    the mask-based form against the efficient path at 32K;
  * ``e2e``: the public host-buffer call with its host<->device copies timed;
  * ``cpu_baseline``: the fp64 oracle on the host cores on a bounded row sample.

Under torchrun (N > 1) every rank runs its own independent replica of the workload
(the path has no cross-GPU exchange: problems shard by sequence and KV-head group),
so scaling is weak; every timed region is bracketed by barriers and its length is the
maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
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
STAGES = ("pool", "gate", "route", "past", "own")
# the long-context workloads timed beside the headline one
SIDE_CONFIGS = ("gqa128k", "varlen")


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


def config_dict(w: synth.Workload, world: int) -> dict:
    """The workload description both arms print (same keys, same values)."""
    q_gb = w.total_tokens * w.num_q_heads * w.head_dim * 2 / 1e9
    return {"workload": workload_desc(w), "seq_len": w.max_seqlen, "global_batch": w.num_seqs * world,
            "total_tokens_per_gpu": w.total_tokens, "parallelism": "replicas%d" % world,
            "l2": "inputs larger than L2 (Q alone %.1f GB)" % q_gb}


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


def dense_causal_flops(w: synth.Workload) -> int:
    """4 D Hq sum_s S_s (S_s + 1) / 2: QK^T and PV over every causal key."""
    return int(sum(4 * w.head_dim * w.num_q_heads * L * (L + 1) // 2 for L in w.seqlens))


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


def kernel_traffic(record: str, units: int):
    """DRAM bytes per launch of an attention kernel, from its committed ncu record (one
    capture at 128K GQA) scaled by the units one launch processes, or None when the kernel's
    sources changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", record)
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
    per_unit = (rec["dram_bytes_read"] + rec["dram_bytes_write"]) / rec["units"]
    return per_unit * units, "scaled from the %s capture by %s" % (rec["workload"], rec["unit_kind"])


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
class MobaPass:
    """Device buffers of one workload and one forward pass through the five C-ABI stages."""

    def __init__(self, w: synth.Workload, dev, host=None, top_k: int | None = None):
        import torch
        import block_sparse_attention_gate_b200 as mb
        self.mb = mb
        self.w = w
        self.dev = dev
        if host is None:
            host = make_host_inputs(w, pinned=False)
        self.Q = host["q"].to(dev)
        self.K = host["k"].to(dev)
        self.V = host["v"].to(dev)
        k = w.top_k if top_k is None else top_k
        self.top_k = k
        self.p = mb.MobaParams(w.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, k)
        self.ws = mb.alloc_workspace(self.p, dev)
        T, hq, _ = self.Q.shape
        self.kbar = torch.empty(self.p.kbar_elems, dtype=torch.float32, device=dev)
        self.sel = torch.empty((T, hq, k), dtype=torch.int32, device=dev)
        self.O = torch.empty_like(self.Q)
        self.LSE = torch.empty((T, hq), dtype=torch.float32, device=dev)

    def step(self, stream, ev=None):
        mb, p = self.mb, self.p
        if ev is not None:
            ev[0].record(stream)
        mb.moba_pool_keys(p, self.K, self.kbar, stream)
        if ev is not None:
            ev[1].record(stream)
        mb.moba_gate_topk(p, self.Q, self.kbar, self.sel, self.ws, stream)
        if ev is not None:
            ev[2].record(stream)
        mb.moba_route(p, self.sel, self.ws, stream)
        if ev is not None:
            ev[3].record(stream)
        mb.moba_attn_past(p, self.Q, self.K, self.V, self.ws, stream)
        if ev is not None:
            ev[4].record(stream)
        mb.moba_attn_self_merge(p, self.Q, self.K, self.V, self.sel, self.ws, self.O, self.LSE, stream)
        if ev is not None:
            ev[5].record(stream)

    def routed_rows(self) -> int:
        if self.top_k < 2:
            return 0
        return int((self.sel[:, :, 1:] >= 0).sum().item())


def time_pass(mp: MobaPass, steps: int, warmup: int, dist, clocks=None) -> dict:
    """W untimed passes, then K passes timed by CUDA events on the launching stream (per
    stage, between barriers and device synchronisations); max over ranks."""
    import torch
    dev = mp.dev
    stream = torch.cuda.current_stream(dev)
    warm = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(warmup):
        mp.step(stream, warm)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    if clocks is not None:
        clocks.start()
    torch.cuda.synchronize(dev)
    for i in range(steps):
        mp.step(stream, evs[i])
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop() if clocks is not None else None
    total_ms = evs[0][0].elapsed_time(evs[-1][5])
    stage_ms = {s: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j, s in enumerate(STAGES)}
    return {"total_ms": max_over_ranks(total_ms, dist, dev), "stage_ms": stage_ms, "clocks": clk}


def attn_fractions(fl: dict, stage_ms: dict, peaks: dict) -> dict:
    attn_s = (stage_ms["past"] + stage_ms["own"]) / 1e3
    attn_tf = fl["attn"] / attn_s / 1e12 if attn_s > 0 else 0.0
    past_tf = fl["past"] / (stage_ms["past"] / 1e3) / 1e12 if stage_ms["past"] > 0 else 0.0
    own_tf = fl["own"] / (stage_ms["own"] / 1e3) / 1e12 if stage_ms["own"] > 0 else 0.0
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    return {"attn_eff_tflops": attn_tf, "attn_frac_of_burst": attn_tf / burst,
            "attn_frac_of_sustained": attn_tf / sus, "past_tflops": past_tf, "own_tflops": own_tf}


def time_side_config(name: str, dev, dist, peaks: dict, steps: int = 3, warmup: int = 3) -> dict:
    """One of the other long-context workloads, timed like the headline one."""
    import torch
    w = synth.CONFIGS[name]
    mp = MobaPass(w, dev)
    t = time_pass(mp, steps, warmup, dist)
    routed = mp.routed_rows()
    fl = flop_counts(w, routed)
    ms = t["total_ms"] / steps
    out = {"workload": workload_desc(w), "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "tokens_per_s": w.total_tokens / (ms / 1e3),
           "eff_tflops": (fl["attn"] + fl["gate"]) / (ms / 1e3) / 1e12,
           "stage_ms": t["stage_ms"], "routed_rows": routed, "flops": fl}
    out.update(attn_fractions(fl, t["stage_ms"], peaks))
    del mp
    torch.cuda.empty_cache()
    return out


def sdpa_dense_causal_ms(Q, K, V, heads_per_call: int, reps: int = 1):
    """Dense causal attention (torch SDPA, cuDNN backend if it accepts the call, else flash,
    else memory-efficient) over [T, H, D] tensors of one sequence.  The inputs are first
    laid out as contiguous [1, H, T, D] with K and V repeated over each GQA group (outside
    the timed region); the calls then run over groups of query heads so that no tensor of
    a call exceeds 2^31 elements.  Returns (ms per whole pass, backend name)."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    T, hq, D = Q.shape
    G = hq // K.shape[1]
    hpc = max(G, heads_per_call - heads_per_call % G)
    q_all = Q.permute(1, 0, 2).contiguous().unsqueeze(0)
    k_all = K.repeat_interleave(G, dim=1).permute(1, 0, 2).contiguous().unsqueeze(0)
    v_all = V.repeat_interleave(G, dim=1).permute(1, 0, 2).contiguous().unsqueeze(0)
    calls = [(q_all[:, h0:h0 + hpc], k_all[:, h0:h0 + hpc], v_all[:, h0:h0 + hpc]) for h0 in range(0, hq, hpc)]

    def run_all(backend):
        with sdpa_kernel([backend]):
            for q, k, v in calls:
                F.scaled_dot_product_attention(q, k, v, is_causal=True)

    result = (None, "no SDPA backend accepted the call")
    for backend, name in ((SDPBackend.CUDNN_ATTENTION, "cudnn"), (SDPBackend.FLASH_ATTENTION, "flash"),
                          (SDPBackend.EFFICIENT_ATTENTION, "efficient")):
        try:
            run_all(backend)  # warm-up (plan build) on the same shapes
            torch.cuda.synchronize()
        except RuntimeError:
            continue
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            run_all(backend)
        b.record()
        torch.cuda.synchronize()
        result = (a.elapsed_time(b) / reps, name)
        break
    del calls, q_all, k_all, v_all
    torch.cuda.empty_cache()
    return result


def dense_comparators(mp_main: MobaPass, main_ms: float, dev, dist) -> dict:
    """Dense causal attention on the same GPU, outside the MoBA timed region."""
    import torch
    res = {}
    w = mp_main.w
    if w.num_seqs == 1:
        ms, backend = sdpa_dense_causal_ms(mp_main.Q, mp_main.K, mp_main.V, heads_per_call=4)
        ms = max_over_ranks(ms if ms is not None else -1.0, dist, dev)
        fl = dense_causal_flops(w)
        res[w.name] = {"impl": "torch SDPA dense causal (%s), heads in groups of 4" % backend,
                       "ms": ms, "flops": fl, "tflops": fl / (ms / 1e3) / 1e12 if ms and ms > 0 else None,
                       "moba_ms": main_ms, "moba_speedup": ms / main_ms if ms and ms > 0 else None}
    # 32K MHA: SDPA, the library in its full mode (top_k = 16 = number of blocks) and MoBA top_k 3
    w32 = synth.CONFIGS["mha32k"]
    host = make_host_inputs(w32, pinned=False)
    full = MobaPass(w32, dev, host=host, top_k=16)
    t_full = time_pass(full, 5, 3, dist)
    ms_sdpa, backend = sdpa_dense_causal_ms(full.Q, full.K, full.V, heads_per_call=32, reps=5)
    ms_sdpa = max_over_ranks(ms_sdpa if ms_sdpa is not None else -1.0, dist, dev)
    del full
    moba = MobaPass(w32, dev, host=host)
    t_moba = time_pass(moba, 5, 3, dist)
    del moba
    torch.cuda.empty_cache()
    fl = dense_causal_flops(w32)
    full_ms = t_full["total_ms"] / 5
    moba_ms = t_moba["total_ms"] / 5
    res["mha32k"] = {"sdpa_impl": "torch SDPA dense causal (%s)" % backend, "sdpa_ms": ms_sdpa,
                     "sdpa_tflops": fl / (ms_sdpa / 1e3) / 1e12 if ms_sdpa > 0 else None,
                     "library_full_ms": full_ms, "library_full_tflops": fl / (full_ms / 1e3) / 1e12,
                     "library_full_stage_ms": t_full["stage_ms"], "flops": fl,
                     "moba_top3_ms": moba_ms, "moba_speedup_vs_sdpa": ms_sdpa / moba_ms if ms_sdpa > 0 else None,
                     "moba_speedup_vs_library_full": full_ms / moba_ms}
    return res


def time_backward(mp: MobaPass, dist, steps: int = 2, warmup: int = 1) -> dict:
    """The backward pass (moba_attn_bwd) at the workload of `mp`, after its forward: selection
    held fixed, dO synthetic N(0,1).  FLOPs by the usual accounting, 2.5x the forward
    attention's (five matrix products against two; the kernels recompute S and dP once more)."""
    import torch
    mb = mp.mb
    stream = torch.cuda.current_stream(mp.dev)
    mp.step(stream)
    dO = torch.randn(mp.Q.shape, dtype=torch.bfloat16, device=mp.dev,
                     generator=torch.Generator(device=mp.dev).manual_seed(7))
    ws = torch.empty(max(mb.moba_bwd_workspace_size(mp.p), 256), dtype=torch.uint8, device=mp.dev)
    dQ, dK, dV = torch.empty_like(mp.Q), torch.empty_like(mp.K), torch.empty_like(mp.V)

    def run():
        mb.moba_attn_bwd(mp.p, mp.Q, mp.K, mp.V, mp.O, mp.LSE, dO, mp.sel, ws, dQ, dK, dV, stream)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize(mp.dev)
    if dist is not None:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        run()
    b.record(stream)
    torch.cuda.synchronize(mp.dev)
    ms = max_over_ranks(a.elapsed_time(b) / steps, dist, mp.dev)
    fl = flop_counts(mp.w, mp.routed_rows())
    bw_flops = int(2.5 * fl["attn"])
    del ws, dQ, dK, dV, dO
    torch.cuda.empty_cache()
    return {"ms": ms, "steps": steps, "warmup": warmup, "flops": bw_flops,
            "tflops": bw_flops / (ms / 1e3) / 1e12, "workload": workload_desc(mp.w),
            "flop_accounting": "2.5 x forward attention FLOPs (S, dP, dV, dK, dQ products)"}


def time_decode(mp: MobaPass, dist, peaks: dict, nseq: int = 8, reps: int = 20) -> dict:
    """Gated decode over the headline workload's keys and values seen as the KV caches of
    `nseq` sequences of equal length (the newest token of each is the query), next to dense
    decode (torch SDPA over every cached key) on the same caches."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    mb, w = mp.mb, mp.w
    T = w.total_tokens
    L = T // nseq
    cu = np.arange(nseq + 1, dtype=np.int32) * L
    p = mb.MobaParams(cu, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.top_k)
    K, V = mp.K[:nseq * L], mp.V[:nseq * L]
    Qd = mp.Q[torch.as_tensor(cu[1:] - 1, device=mp.dev, dtype=torch.long)].contiguous()
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device=mp.dev)
    mb.moba_pool_keys(p, K, kbar)
    ws = torch.empty(max(mb.moba_decode_workspace_size(p), 256), dtype=torch.uint8, device=mp.dev)
    sel = torch.empty((nseq, w.num_q_heads, w.top_k), dtype=torch.int32, device=mp.dev)
    O = torch.empty_like(Qd)
    LSE = torch.empty((nseq, w.num_q_heads), dtype=torch.float32, device=mp.dev)
    stream = torch.cuda.current_stream(mp.dev)

    def timed(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(mp.dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize(mp.dev)
        return a.elapsed_time(b) / n

    ms = timed(lambda: mb.moba_decode_fwd(p, Qd, K, V, kbar, ws, O, LSE, sel=sel, stream=stream), reps)
    ms = max_over_ranks(ms, dist, mp.dev)
    # algorithmic bytes: the distinct selected blocks' keys and values per (sequence, KV head)
    # (the own block up to the new token), the pooled keys the gate reads, Q and O
    s_np = sel.cpu().numpy()
    G, bs, D = w.num_q_heads // w.num_kv_heads, w.block_size, w.head_dim
    own = (L - 1) // bs
    nbytes = 0
    for sq in range(nseq):
        for g in range(w.num_kv_heads):
            blocks = set(int(b) for b in s_np[sq, g * G:(g + 1) * G].ravel() if b >= 0)
            for b in blocks:
                nbytes += (L - b * bs if b == own else bs) * D * 2 * 2
    nbytes += nseq * w.num_kv_heads * own * D * 4 + 2 * Qd.numel() * 2
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    res = {"workload": "%d sequences x %d cached tokens, Hq=%d Hkv=%d D=%d block_size=%d top_k=%d (the headline "
                       "workload's keys and values)" % (nseq, L, w.num_q_heads, w.num_kv_heads, D, bs, w.top_k),
           "ms": ms, "tokens_per_s": nseq / (ms / 1e3), "algorithmic_bytes": nbytes,
           "achieved_gbs": nbytes / (ms / 1e3) / 1e9, "hbm_peak_gbs": hbm,
           "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / hbm, "launches": 3}
    # dense decode: every cached key, torch SDPA (one query per sequence and head)
    q4 = Qd.unsqueeze(2)  # [B, Hq, 1, D]
    k4 = K.view(nseq, L, w.num_kv_heads, D).permute(0, 2, 1, 3)
    v4 = V.view(nseq, L, w.num_kv_heads, D).permute(0, 2, 1, 3)
    k4 = k4.repeat_interleave(G, dim=1).contiguous()
    v4 = v4.repeat_interleave(G, dim=1).contiguous()
    dense = None
    for backend, name in ((SDPBackend.CUDNN_ATTENTION, "cudnn"), (SDPBackend.FLASH_ATTENTION, "flash"),
                          (SDPBackend.EFFICIENT_ATTENTION, "efficient")):
        try:
            with sdpa_kernel([backend]):
                dms = timed(lambda: F.scaled_dot_product_attention(q4, k4, v4), reps)
            dense = (max_over_ranks(dms, dist, mp.dev), name)
            break
        except RuntimeError:
            continue
    if dense is not None:
        dbytes = 2 * nseq * w.num_kv_heads * L * D * 2
        res["dense_decode"] = {"impl": "torch SDPA (%s) over every cached key" % dense[1], "ms": dense[0],
                               "kv_bytes_per_kv_head": dbytes, "moba_speedup": dense[0] / ms}
    del k4, v4, ws, kbar
    torch.cuda.empty_cache()
    return res


def time_mask_based(dev, dist) -> dict:
    """The mask-based form (moba_attn_naive: every causal key scored, unselected blocks
    masked) against the efficient path (route + past blocks + own block), on the same
    selection: at 32K tokens with one head, block 2048, top_k 3 (the configuration of the
    pages' efficient-versus-naive comparison) and at 32K MHA (32 heads)."""
    import torch
    out = {}
    for name, w in (("32k_1head", synth.Workload("mask32k_h1", [32768], 1, 1, 128, 2048, 3, seed=1006,
                                                 rope_theta=500000.0)),
                    ("mha32k", synth.CONFIGS["mha32k"])):
        mp = MobaPass(w, dev)
        stream = torch.cuda.current_stream(dev)
        mb, p = mp.mb, mp.p
        mp.step(stream)
        On, Ln = torch.empty_like(mp.O), torch.empty_like(mp.LSE)

        def timed(fn, n=10):
            for _ in range(3):
                fn()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) / n

        eff = timed(lambda: mb.moba_attn_fwd(p, mp.Q, mp.K, mp.V, mp.sel, mp.ws, mp.O, mp.LSE, stream))
        nv = timed(lambda: mb.moba_attn_naive(p, mp.Q, mp.K, mp.V, mp.sel, On, Ln, stream))
        eff, nv = max_over_ranks(eff, dist, dev), max_over_ranks(nv, dist, dev)
        out[name] = {"workload": workload_desc(w), "efficient_ms": eff, "mask_based_ms": nv,
                     "speedup": nv / eff, "dense_causal_flops": dense_causal_flops(w),
                     "mask_based_tflops": dense_causal_flops(w) / (nv / 1e3) / 1e12}
        del mp, On, Ln
        torch.cuda.empty_cache()
    return out


def time_10m_group(dev, dist, peaks: dict, steps: int = 2, warmup: int = 1) -> dict:
    """A 10M-token prefill: one sequence of 10,485,760 tokens with one KV-head group of the
    Llama shape (4 query heads on 1 KV head, D 128, block 2048, top_k 3, rotary inputs with
    planted relevance).  The full 32/8-head problem does not fit one GPU (Q alone is 86 GB)
    and runs group by group; its time is 8 times this group's (the groups are independent)."""
    import torch
    w = synth.Workload("prefill10m_group", [10 * 1048576], 4, 1, 128, 2048, 3, seed=1010,
                       rope_theta=500000.0, plant=0.5)
    mp = MobaPass(w, dev)
    t = time_pass(mp, steps, warmup, dist)
    routed = mp.routed_rows()
    fl = flop_counts(w, routed)
    ms = t["total_ms"] / steps
    out = {"workload": workload_desc(w), "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "tokens_per_s": w.total_tokens / (ms / 1e3), "stage_ms": t["stage_ms"], "routed_rows": routed,
           "flops": fl, "eff_tflops": (fl["attn"] + fl["gate"]) / (ms / 1e3) / 1e12,
           "full_heads_32_8_ms_estimate": 8 * ms,
           "full_heads_tokens_per_s_estimate": w.total_tokens / (8 * ms / 1e3)}
    out.update(attn_fractions(fl, t["stage_ms"], peaks))
    del mp
    torch.cuda.empty_cache()
    return out


def run_ours(args, w: synth.Workload, rank: int, world: int, dist) -> dict | None:
    import torch
    import block_sparse_attention_gate_b200 as mb

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    host = make_host_inputs(w, pinned=True, nthreads=max(1, (os.cpu_count() or 1) // world))
    mp = MobaPass(w, dev, host=host)
    peaks, peak_kind = load_peaks()
    clocks = ClockSampler(local)
    t = time_pass(mp, args.steps, args.warmup, dist, clocks)
    stage_ms, clk = t["stage_ms"], t["clocks"]
    t_max = t["total_ms"]
    routed = mp.routed_rows()
    fl = flop_counts(w, routed)
    ms_step = t_max / args.steps
    T = w.total_tokens
    tokens_per_s = job_throughput(T, world, args.steps, t_max)

    # ----- end to end through the public call with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        # the public host-buffer call: per-KV-group slices copied and computed over 3 streams
        O_host = torch.empty(mp.O.shape, dtype=torch.bfloat16, pin_memory=True)
        L_host = torch.empty(mp.LSE.shape, dtype=torch.float32, pin_memory=True)
        streams = [torch.cuda.Stream(dev) for _ in range(3)]
        staging = torch.empty(max(mb.moba_host_staging_size(mp.p, len(streams)), 256), dtype=torch.uint8,
                              device=dev)
        n_e2e = max(1, min(args.steps, 3))
        main_stream = torch.cuda.current_stream(dev)

        def e2e_run(n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(main_stream)
            for s_ in streams:
                s_.wait_event(a)
            for _ in range(n):
                mb.moba_fwd_host(mp.p, host["q"], host["k"], host["v"], O_host, L_host, staging, streams)
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
        d2h = mp.O.numel() * 2 + mp.LSE.numel() * 4
        e2e = {"value": job_throughput(T, world, n_e2e, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e}
        del staging, streams
        torch.cuda.empty_cache()

    traffic, traffic_note = kernel_traffic("attn_past_traffic.json", routed)
    own_traffic, own_note = kernel_traffic("attn_own_traffic.json", T * w.num_q_heads)
    peak_tf = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    past_s = stage_ms["past"] / 1e3
    achieved = fl["past"] / past_s / 1e12 if past_s > 0 else 0.0
    own_s = stage_ms["own"] / 1e3
    own_achieved = fl["own"] / own_s / 1e12 if own_s > 0 else 0.0
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
        "config": config_dict(w, world),
        "eff_tflops": eff_tf,
        "pct_bf16_peak": 100.0 * eff_tf / peak_tf,
        "stage_ms": stage_ms,
        "flops": fl,
        "routed_rows": routed,
        "roofline": {"bound": "tensor", "kernel": "past-block attention", "achieved": achieved,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                     "peak_kind": "%s bf16 sustained (kernel timed inside a long step)" % peak_kind,
                     "traffic": traffic, "traffic_note": traffic_note},
        # the second attention kernel (own block + merge, with the partial pre-merge when used)
        "roofline_own": {"bound": "tensor", "kernel": "own block + merge", "achieved": own_achieved,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": own_achieved / peak_tf,
                         "peak_kind": "%s bf16 sustained" % peak_kind,
                         "traffic": own_traffic, "traffic_note": own_note},
        "clocks": clk,
        "gpu_launches": mb.moba_launches_per_forward(mp.p) * args.steps,
        "e2e": e2e,
    }
    res.update(attn_fractions(fl, stage_ms, peaks))
    res["peaks"] = {"bf16_burst": peaks.get("bf16_tflops"), "bf16_sustained": peak_tf, "kind": peak_kind}
    if not args.no_side:
        res["configs"] = {name: time_side_config(name, dev, dist, peaks) for name in SIDE_CONFIGS
                          if name != w.name}
    if not args.no_dense:
        res["dense_causal"] = dense_comparators(mp, ms_step, dev, dist)
    if not args.no_extra:
        res["backward"] = time_backward(mp, dist)
        res["decode"] = time_decode(mp, dist, peaks)
        res["mask_based"] = time_mask_based(dev, dist)
    if not args.no_10m:
        res["prefill10m_group"] = time_10m_group(dev, dist, peaks)
    if rank == 0 and world == 1 and not args.no_cpu:
        Kh = host["k"].view(torch.int16).numpy().view(np.uint16)
        Vh = host["v"].view(torch.int16).numpy().view(np.uint16)
        tps, nrows, secs, thr, pool_s = oracle_rows_per_second(w, Kh, Vh, args.cpu_seconds)
        res["cpu_baseline"] = {
            "value": tps, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": "%d random query rows of the same workload in %.1f s plus one pooling pass over "
                      "all keys (%.1f s); per-row time extrapolated to all T*Hq rows" % (nrows, secs, pool_s)}
    return res


def run_reference(args, w: synth.Workload, rank: int, world: int) -> dict | None:
    """The oracle (fp64 CPU, all host cores) on a bounded sample of the same workload.

    Each step is one bounded sample (about --ref-seconds of oracle rows plus one pooling
    pass over all keys); ``ms_per_step`` is that measured step time, and ``value`` the
    throughput it implies for the whole pass (tokens/s, per-row time extrapolated to every
    row).  The extrapolated time of one whole pass is reported separately."""
    if rank != 0:
        return None
    Kh = w.fill("k")
    Vh = w.fill("v")
    vals, rows_all, secs_all, step_s = [], 0, 0.0, []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        tps, nrows, secs, thr, pool_s = oracle_rows_per_second(w, Kh, Vh, args.ref_seconds, seed=i)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            vals.append(tps)
            rows_all += nrows
            secs_all += secs
            step_s.append(dt)
    v = statistics.mean(vals)
    T = w.total_tokens
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(step_s),
        "ms_per_full_pass_extrapolated": 1e3 * T / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded splitmix64/Box-Muller normals, RoPE, planted relevance per recipe)",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": "%d random query rows over %d steps (%.1f s of rows) plus one pooling "
                                   "pass per step, extrapolated to all rows" % (rows_all, args.steps, secs_all)},
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
    ap.add_argument("--no-side", action="store_true", help="skip the other long-context workloads")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense causal comparators")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the backward, decode and mask-based records")
    ap.add_argument("--no-10m", action="store_true", help="skip the 10M-token (one KV-head group) record")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="scale the workload's sequence lengths (for small profiling captures)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=4.0)
    args = ap.parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = synth.CONFIGS[args.config]
    if args.scale != 1.0:
        import dataclasses
        lens = [max(1, int(round(L * args.scale))) for L in w.seqlens]
        w = dataclasses.replace(w, name="%s_x%g" % (w.name, args.scale), seqlens=lens)
    if args.impl == "reference":
        res = run_reference(args, w, rank, world)
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
