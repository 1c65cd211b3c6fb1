"""Gate ties on the GPU, checked row by row against the fp64 oracle with the order included.

The gate takes the top_k - 1 earlier blocks with the largest <q, Kbar[b]> (MoBA README,
"Parameter-less Gating Mechanism"), ties to the lower block index (the library's contract).
Here every key of block b is c_b * u, with c_b a power of two from a short cycle and u one
fixed bf16 vector per KV head, so Kbar[b] = c_b * u exactly: many blocks share a pooled key
and score exactly alike, and the others differ by a factor of two.  Every selection, order
included, is therefore fixed, and the library must return the oracle's on every row whose
query is not nearly orthogonal to u: rows with |<q, u>| < 1e-3 |q| |u| put every score
near zero, where blocks c and c/2 are no longer apart at the gate's resolution (the parity
rule's 1e-3 relative gap), and are left out (a handful of rows).  More
than 64 blocks make the gate walk several candidate chunks and groups, so ties fall inside
a 32-block group, across groups and across chunks; top_k 3, 5 and 9 cover the quantized
selection for two and four blocks and the exact one for eight.
"""
import numpy as np
import pytest

import oracle
import synth
from _harness import params, problem, to_device_bf16

pytestmark = pytest.mark.gpu

CYCLE = np.array([1.0, 0.5, 1.0, 0.25, 0.5, 1.0, 0.125, 1.0, 2.0 ** -4], dtype=np.float32)


def tied_inputs(w: synth.Workload):
    Q = w.fill("q")
    u = synth.bf16_bits_to_f32(w.fill("k", 0, 1))[0]  # [Hkv, D]
    T = w.total_tokens
    c = np.empty(T, dtype=np.float32)
    for s in range(w.num_seqs):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        blk = np.arange(b - a) // w.block_size
        c[a:b] = CYCLE[blk % CYCLE.size]
    K = synth.f32_to_bf16_bits(c[:, None, None] * u[None])
    return Q, K


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("top_k", [3, 5, 9])
def test_gate_ties_match_oracle_exactly(D, top_k, cuda_device):
    import torch
    import block_sparse_attention_gate_b200 as mb
    w = synth.Workload("ties_%d_%d" % (D, top_k), [128 * 150 + 77, 128 * 40 + 5], 4, 2, D, 128, top_k,
                       seed=300 + D + top_k)
    Q, K = tied_inputs(w)
    p = params(w)
    T, hq, _ = Q.shape
    Qd, Kd = to_device_bf16(Q), to_device_bf16(K)
    ws = mb.alloc_workspace(p)
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device="cuda")
    sel = torch.empty((T, hq, top_k), dtype=torch.int32, device="cuda")
    mb.moba_pool_keys(p, Kd, kbar)
    mb.moba_gate_topk(p, Qd, kbar, sel, ws)
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    got = sel.cpu().numpy()
    pr = problem(w)
    kb = oracle.pool_keys(pr, K)
    tt, hh = np.meshgrid(np.arange(T, dtype=np.int64), np.arange(hq, dtype=np.int32), indexing="ij")
    ref = oracle.rows(pr, Q.reshape(T * hq, D), None, None, kb, tt.ravel(), hh.ravel(),
                      attention=False)["sel"].reshape(T, hq, top_k)
    qf = synth.bf16_bits_to_f32(Q).astype(np.float64)
    uf = synth.bf16_bits_to_f32(w.fill("k", 0, 1))[0].astype(np.float64)
    G = hq // w.num_kv_heads
    uh = uf[np.arange(hq) // G]  # [hq, D]
    cos = np.einsum("thd,hd->th", qf, uh) / (np.linalg.norm(qf, axis=2) * np.linalg.norm(uh, axis=1) + 1e-300)
    keep = np.abs(cos) >= 1e-3
    assert keep.mean() > 0.99
    bad = np.argwhere((got != ref).any(axis=2) & keep)
    assert bad.size == 0, (len(bad), bad[:5].tolist(),
                           [(got[t, h].tolist(), ref[t, h].tolist()) for t, h in bad[:5]])
