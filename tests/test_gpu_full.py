"""GPU parity at the full workload sizes, in the launch configuration the benchmark times
(one moba_fwd call per pass), on a seeded sample of query rows that the fp64 oracle
computes one by one: per sequence and KV-head group 4096 random tokens plus the first and
last token of every block, each with all the group's query heads.  (The 32K MHA workload
is checked on every row, in its own file.)"""
import numpy as np
import pytest

import oracle
import synth
from _harness import assert_parity, compare, kbar_seq_order, problem, run_gpu, sample_rows, KBAR_ABS

pytestmark = pytest.mark.gpu

PER_GROUP = 4096


def check_structure(w, sel):
    """Every row, not only the sample: own block in slot 0, padding -1, past blocks only."""
    for s in range(w.num_seqs):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        own = ((np.arange(a, b) - a) // w.block_size)[:, None]
        ss = sel[a:b]
        assert np.all(ss[:, :, 0] == own)
        if w.top_k > 1:
            past = ss[:, :, 1:]
            m = np.minimum(w.top_k - 1, own)[:, :, None]
            slot = np.arange(w.top_k - 1)[None, None, :]
            assert np.all((past >= 0) == (slot < m))
            assert np.all(past < own[:, :, None])
            # chosen past blocks are distinct
            srt = np.sort(past, axis=-1)
            assert not np.any((srt[:, :, 1:] == srt[:, :, :-1]) & (srt[:, :, 1:] >= 0))


@pytest.mark.parametrize("name", ["gqa128k", "varlen", "prefill1m"])
def test_full_size_workload_sampled_rows(name, cuda_device):
    w = synth.CONFIGS[name]
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    gpu = run_gpu(w, Q, K, V)
    pr = problem(w)
    kbar = oracle.pool_keys(pr, K)
    np.testing.assert_allclose(kbar_seq_order(w, gpu["Kbar"]), kbar, rtol=0, atol=KBAR_ABS)
    tok, hd = sample_rows(w, PER_GROUP, seed=1)
    orc = oracle.rows(pr, Q[tok, hd], K, V, kbar, tok, hd)
    st = compare(gpu["sel"][tok, hd], gpu["O"][tok, hd], gpu["LSE"][tok, hd], orc)
    print(name, st)
    assert_parity(st)
    check_structure(w, gpu["sel"])
    assert np.isfinite(gpu["O"]).all() and np.isfinite(gpu["LSE"]).all()
