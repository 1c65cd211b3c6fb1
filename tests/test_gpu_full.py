"""GPU parity at the full workload sizes, in the launch configuration the benchmark times
(one moba_fwd call per pass), on a seeded sample of query rows that the fp64 oracle
computes one by one: per KV-head group a random spread of tokens plus the first and last
token of every block, each with all the group's query heads."""
import numpy as np
import pytest

import oracle
import synth
from _harness import assert_parity, compare, kbar_seq_order, problem, run_gpu, sample_rows, KBAR_ABS

pytestmark = pytest.mark.gpu

# per-group random rows; the 1M case follows the 4096-rows-per-group recipe
PER_GROUP = {"mha32k": 512, "gqa128k": 1024, "prefill1m": 4096, "varlen": 512}


@pytest.mark.parametrize("name", ["mha32k", "gqa128k", "varlen", "prefill1m"])
def test_full_size_workload_sampled_rows(name, cuda_device):
    w = synth.CONFIGS[name]
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    gpu = run_gpu(w, Q, K, V)
    pr = problem(w)
    kbar = oracle.pool_keys(pr, K)
    np.testing.assert_allclose(kbar_seq_order(w, gpu["Kbar"]), kbar, rtol=0, atol=KBAR_ABS)
    tok, hd = sample_rows(w, PER_GROUP[name], seed=1)
    orc = oracle.rows(pr, Q[tok, hd], K, V, kbar, tok, hd)
    st = compare(gpu["sel"][tok, hd], gpu["O"][tok, hd], gpu["LSE"][tok, hd], orc)
    print(name, st)
    assert_parity(st)
    # every row, not only the sample: own block in slot 0, padding -1, distinct past blocks
    sel = gpu["sel"]
    for s in range(w.num_seqs):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        own = ((np.arange(a, b) - a) // w.block_size)[:, None]
        ss = sel[a:b]
        assert np.all(ss[:, :, 0] == own)
        past = ss[:, :, 1:]
        m = np.minimum(w.top_k - 1, own)[:, :, None] if w.top_k > 1 else None
        if m is not None:
            slot = np.arange(w.top_k - 1)[None, None, :]
            assert np.all((past >= 0) == (slot < m))
            assert np.all(past < own[:, :, None])
    assert np.isfinite(gpu["O"]).all() and np.isfinite(gpu["LSE"]).all()
