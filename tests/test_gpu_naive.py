"""GPU parity of the mask-based attention (moba_attn_naive: every causal key scored, keys
outside the selected blocks masked) against the fp64 oracle, on the selection the library's
gate made, and its agreement with the efficient path (moba_attn_fwd) on the same selection."""
import numpy as np
import pytest

import oracle
import synth
from _harness import assert_parity, compare, params, problem, run_gpu, to_device_bf16

pytestmark = pytest.mark.gpu

CASES = [
    synth.Workload("nv_ragged_gqa", [1000, 333, 2125, 128, 1], 4, 2, 128, 128, 3, seed=51,
                   rope_theta=500000.0, plant=0.5),
    synth.Workload("nv_d64", [777, 1536], 8, 1, 64, 256, 4, seed=52, rope_theta=10000.0),
    synth.Workload("nv_gqa_odd", [1500, 640], 6, 2, 128, 256, 3, seed=53, rope_theta=500000.0),
    synth.Workload("nv_top1", [600, 300], 2, 2, 128, 128, 1, seed=54),
    synth.Workload("nv_full", [640], 4, 1, 128, 128, 16, seed=55),
    synth.Workload("nv_k8_chunks", [9300], 2, 1, 128, 128, 8, seed=56, plant=0.5),
    synth.Workload("nv_empty", [300, 0, 700, 0, 129], 4, 2, 64, 128, 3, seed=57),
    synth.Workload("nv_bs2048", [5000], 4, 4, 128, 2048, 2, seed=58, rope_theta=500000.0),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_mask_based_attention_matches_oracle(w, cuda_device):
    import torch
    import block_sparse_attention_gate_b200 as mb
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    eff = run_gpu(w, Q, K, V)
    p = params(w)
    Qd, Kd, Vd = to_device_bf16(Q), to_device_bf16(K), to_device_bf16(V)
    sel = torch.from_numpy(eff["sel"]).cuda()
    O = torch.full_like(Qd, float("nan"))
    LSE = torch.full((w.total_tokens, w.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    mb.moba_attn_naive(p, Qd, Kd, Vd, sel, O, LSE)
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    On, Ln = O.float().cpu().numpy(), LSE.cpu().numpy()
    orc = oracle.full(problem(w), Q, K, V)
    st = compare(eff["sel"], On, Ln, orc)
    print(w.name, st)
    assert_parity(st)
    # the two forms agree with each other to within the bf16 rounding of the outputs
    assert np.all(np.abs(On - eff["O"]) <= 1e-2 + 2.0 ** -8 * np.abs(eff["O"]))
    assert np.max(np.abs(Ln - eff["LSE"])) <= 1e-3
