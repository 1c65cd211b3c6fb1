"""GPU parity of the MoBA backward pass (moba_attn_bwd) against the fp64 oracle
(oracle.backward: gradients of masked softmax attention under the forward's selection).

The selection is the oracle's own (a valid selection by the library's contract): the
library's forward (moba_attn_fwd) runs on it and its O and LSE feed the backward, as in a
training step.  The gradients therefore do not depend on how near-tie gate scores fall.

Tolerance (bf16 gradients, fp32 accumulation, P and dS rounded to bf16 for the tensor
cores): each element within 2e-2 + 2^-7 |g| of the fp64 gradient (the output's own
rounding is half an ulp, 2^-8 |g| at most; the rounding of P and dS adds up to 2^-9 of the
sum of the absolute terms), and the relative Frobenius error of each tensor within 1e-2.
"""
import numpy as np
import pytest

import oracle.backward as obw
import synth
from _harness import params, problem, to_device_bf16

pytestmark = pytest.mark.gpu

ABS = 2e-2
REL = 2.0 ** -7
FRO = 1e-2

CASES = [
    synth.Workload("bw_gqa", [1000, 333, 700], 4, 2, 128, 128, 3, seed=71, rope_theta=500000.0, plant=0.5),
    synth.Workload("bw_d64", [777, 1024], 8, 2, 64, 128, 4, seed=72, plant=0.5),
    synth.Workload("bw_odd_g", [1500], 6, 2, 128, 256, 3, seed=73, plant=0.5),
    synth.Workload("bw_top1", [600, 300], 2, 2, 128, 128, 1, seed=74),
    synth.Workload("bw_full", [640], 4, 1, 128, 128, 16, seed=75),
    synth.Workload("bw_k8", [2000], 2, 1, 128, 128, 8, seed=76, plant=0.5),
    synth.Workload("bw_empty", [300, 0, 129, 1], 4, 2, 64, 128, 3, seed=77, plant=0.5),
]


def grad_output(w):
    """The upstream gradient dO: N(0,1) bf16 from the input generator, on a seed of its own."""
    g = synth.Workload(w.name + "_dO", list(w.seqlens), w.num_q_heads, w.num_kv_heads, w.head_dim,
                       w.block_size, w.top_k, seed=w.seed + 5000)
    return g.fill("q")


def stats(got, ref):
    err = np.abs(got - ref)
    return {"max_err": float(err.max()) if err.size else 0.0,
            "over": float((err - (ABS + REL * np.abs(ref))).max()) if err.size else -1.0,
            "fro": float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)),
            "ref_max": float(np.abs(ref).max()) if ref.size else 0.0}


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w, cuda_device):
    import torch
    import block_sparse_attention_gate_b200 as mb
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    dO = grad_output(w)
    pr = problem(w)
    ref = obw.backward(pr, Q, K, V, synth.bf16_bits_to_f32(dO).astype(np.float64))
    p = params(w)
    dev = lambda a: to_device_bf16(a)
    Qd, Kd, Vd, dOd = dev(Q), dev(K), dev(V), dev(dO)
    T, hq, D = Q.shape
    seld = torch.from_numpy(np.ascontiguousarray(ref["sel"], dtype=np.int32)).cuda()
    Od = torch.empty_like(Qd)
    Ld = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    fws = mb.alloc_workspace(p)
    mb.moba_attn_fwd(p, Qd, Kd, Vd, seld, fws, Od, Ld)
    ws = torch.empty(max(mb.moba_bwd_workspace_size(p), 256), dtype=torch.uint8, device="cuda")
    dQ = torch.full_like(Qd, float("nan"))
    dK = torch.full_like(Kd, float("nan"))
    dV = torch.full_like(Vd, float("nan"))
    mb.moba_attn_bwd(p, Qd, Kd, Vd, Od, Ld, dOd, seld, ws, dQ, dK, dV)
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    res = {}
    for name, got in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), name
        res[name] = stats(g, ref[name])
    print(w.name, res)
    for name, st in res.items():
        assert st["over"] <= 0.0, (name, st)
        assert st["fro"] <= FRO, (name, st)
