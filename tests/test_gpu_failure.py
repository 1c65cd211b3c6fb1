"""Failure detection without a GPU fault: a kernel wait that can never complete gives up
after its limit, reports through the device error word and returns; the context stays
usable and the next forward pass runs clean."""
import pytest

import synth
from _harness import assert_parity, compare, problem, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives(cuda_device):
    import oracle
    import block_sparse_attention_gate_b200 as mb
    assert mb.moba_read_device_error(clear=True) == 0
    assert mb.moba_selftest_bounded_wait() == 1
    assert mb.moba_read_device_error() == 0
    w = synth.Workload("after_timeout", [700], 4, 2, 128, 128, 3, seed=31)
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    gpu = run_gpu(w, Q, K, V)  # asserts the error word stays 0
    assert_parity(compare(gpu["sel"], gpu["O"], gpu["LSE"], oracle.full(problem(w), Q, K, V)))
