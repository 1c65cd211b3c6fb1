"""GPU parity of the 32K MHA workload (one sequence of 32768 tokens, 32 query and KV heads,
D 128, block 2048, top_k 3, rotary inputs) against the fp64 oracle on EVERY (token, head)
row: 1,048,576 rows, the oracle's whole pass on the host cores."""
import numpy as np
import pytest

import oracle
import synth
from _harness import assert_parity, compare, kbar_seq_order, problem, run_gpu, KBAR_ABS
from test_gpu_full import check_structure

pytestmark = pytest.mark.gpu


def test_mha32k_every_row(cuda_device):
    w = synth.CONFIGS["mha32k"]
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    gpu = run_gpu(w, Q, K, V)
    orc = oracle.full(problem(w), Q, K, V)
    np.testing.assert_allclose(kbar_seq_order(w, gpu["Kbar"]), orc["Kbar"], rtol=0, atol=KBAR_ABS)
    st = compare(gpu["sel"], gpu["O"], gpu["LSE"], orc)
    print("mha32k all rows", st)
    assert st["rows"] == w.total_tokens * w.num_q_heads
    assert_parity(st)
    check_structure(w, gpu["sel"])
