"""Shared helpers of the GPU parity tests: run the library on a seeded workload and
compare it with the fp64 oracle under the parity rule.

Parity rule (MoBA prefill, bf16 inputs, fp32 accumulation):
  * selected block sets identical on every row whose gap (last chosen minus best
    unchosen gate score) exceeds 1e-3 * max |score| over its candidates;
  * on rows whose selection matches: O within max-abs 1e-2 and mean-abs 1e-3,
    LSE within 1e-3 (absolute).  O is a bf16 output, whose own resolution is coarser than
    1e-2 for |O| >= 2 (an ulp there is 2^-6), so an element may also differ by one bf16
    ulp of the exact value: |O_gpu - O| <= max(1e-2, ulp_bf16(|O|)).  The ulp budget:
    the output's own rounding (half an ulp) plus the bf16 rounding of the probabilities in
    the P V product (up to 2^-9 sum_j P_j |V_j|, up to half an ulp more when a few keys
    dominate a row), the fp16 partials (2^-11) and the fp32 accumulation.  The statistics
    count the elements that the widened bound covers and the ones that needed it;
  * rows whose selection may legitimately differ (gap under the threshold) are
    excluded from the O/LSE comparison and counted.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

SEL_REL_GAP = 1e-3
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 1e-3
# Kbar: fp32 sums of at most 8192 bf16 values of magnitude below ~10; observed errors are ~1e-6
KBAR_ABS = 1e-4


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits; subnormal range not needed here)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7.0)


def problem(w: synth.Workload) -> oracle.Problem:
    return oracle.Problem(w.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                          w.block_size, w.top_k, dtype="bf16")


def to_device_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def params(w: synth.Workload):
    import block_sparse_attention_gate_b200 as mb
    return mb.MobaParams(w.cu_seqlens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                         w.top_k)


def run_gpu(w: synth.Workload, Q: np.ndarray, K: np.ndarray, V: np.ndarray, stages: bool = False) -> dict:
    """Run the library (moba_fwd, or the three entry points when ``stages``) on host inputs."""
    import torch
    import block_sparse_attention_gate_b200 as mb
    p = params(w)
    Qd, Kd, Vd = to_device_bf16(Q), to_device_bf16(K), to_device_bf16(V)
    T, hq, D = Q.shape
    ws = mb.alloc_workspace(p)
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device="cuda")
    sel = torch.empty((T, hq, w.top_k), dtype=torch.int32, device="cuda")
    O = torch.empty_like(Qd)
    LSE = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    if stages:
        mb.moba_pool_keys(p, Kd, kbar)
        mb.moba_gate_topk(p, Qd, kbar, sel, ws)
        mb.moba_attn_fwd(p, Qd, Kd, Vd, sel, ws, O, LSE)
    else:
        mb.moba_fwd(p, Qd, Kd, Vd, ws, O, LSE, Kbar=kbar, sel=sel)
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0, "a kernel wait gave up"
    return {
        "Kbar": kbar.view(w.num_seqs, p.max_blocks, w.num_kv_heads, D).cpu().numpy(),
        "sel": sel.cpu().numpy(),
        "O": O.float().cpu().numpy(),
        "LSE": LSE.cpu().numpy(),
    }


def kbar_seq_order(w: synth.Workload, kbar_padded: np.ndarray) -> np.ndarray:
    """[num_seqs, MB, Hkv, D] -> the oracle's sequence-ordered [NB, Hkv, D]."""
    parts = [kbar_padded[s, :w.blocks_of(s)] for s in range(w.num_seqs)]
    return np.concatenate(parts, axis=0)


def compare(gpu_sel, gpu_O, gpu_LSE, orc: dict) -> dict:
    """Apply the parity rule to matching row lists; returns statistics (asserts nothing).

    Selections are compared as sets (the attention output depends on the set only); rows
    whose set matches but whose descending-score order differs are counted separately
    (two chosen blocks whose scores agree to fp32 rounding may swap places)."""
    sel_o = orc["sel"]
    gap, gmax = orc["gap"], orc["gmax"]
    qualified = gap > SEL_REL_GAP * gmax
    same = np.all(np.sort(gpu_sel, axis=-1) == np.sort(sel_o, axis=-1), axis=-1)
    same_order = np.all(gpu_sel == sel_o, axis=-1)
    bad_sel = int(np.sum(qualified & ~same))
    d_o = np.abs(gpu_O.astype(np.float64) - orc["O"])[same]
    d_l = np.abs(gpu_LSE.astype(np.float64) - orc["lse"])[same]
    wide = bf16_ulp(orc["O"][same])
    tol_o = np.maximum(O_MAX_ABS, wide)
    return {
        "rows": int(same.size),
        "bad_sel": bad_sel,
        "order_swaps": int(np.sum(same & ~same_order)),
        "excluded": int(np.sum(~same)),
        "o_max": float(d_o.max()) if d_o.size else 0.0,
        "o_over": float((d_o - tol_o).max()) if d_o.size else -1.0,
        "o_mean": float(d_o.mean()) if d_o.size else 0.0,
        "o_wide_elems": int(np.sum(wide > O_MAX_ABS)),
        "o_wide_used": int(np.sum((d_o > O_MAX_ABS) & (d_o <= tol_o))),
        "lse_max": float(d_l.max()) if d_l.size else 0.0,
    }


def assert_parity(st: dict, max_excluded_frac: float = 0.01):
    assert st["bad_sel"] == 0, st
    assert st["order_swaps"] <= 1e-3 * st["rows"], st
    assert st["excluded"] <= max_excluded_frac * st["rows"], st
    assert st["o_over"] <= 0.0, st
    assert st["o_mean"] <= O_MEAN_ABS, st
    assert st["lse_max"] <= LSE_ABS, st


def sample_rows(w: synth.Workload, per_group: int, seed: int = 0):
    """Seeded row sample: per (sequence, KV-head group) `per_group` tokens spread over the
    sequence plus the first and last token of every block, each with all G query heads."""
    rng = np.random.default_rng(seed)
    G = w.num_q_heads // w.num_kv_heads
    toks, heads = [], []
    for s in range(w.num_seqs):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        if b == a:
            continue
        edges = []
        for blk in range(w.blocks_of(s)):
            lo = a + blk * w.block_size
            edges += [lo, min(b, lo + w.block_size) - 1]
        for g in range(w.num_kv_heads):
            t = np.unique(np.concatenate([rng.integers(a, b, size=per_group), np.array(edges)]))
            for hh in range(G):
                toks.append(t)
                heads.append(np.full(t.size, g * G + hh))
    return np.concatenate(toks).astype(np.int64), np.concatenate(heads).astype(np.int32)
