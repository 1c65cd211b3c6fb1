"""GPU parity of the whole path (pool, gate, route, block attention, merge) against the
fp64 oracle on every row of small seeded workloads that span several tiles, ragged
sequence tails and the method's degenerate cases."""
import numpy as np
import pytest

import oracle
import synth
from _harness import (KBAR_ABS, assert_parity, compare, kbar_seq_order, problem, run_gpu)

pytestmark = pytest.mark.gpu

SMALL = {
    # the tiny fp32-drawn case (inputs rounded to bf16 for the library)
    "tiny": synth.CONFIGS["tiny"],
    # ragged varlen GQA with rotary and planted relevance; a 1-token and a 1-block sequence
    "ragged_gqa": synth.Workload("ragged_gqa", [1000, 333, 2125, 128, 1], 4, 2, 128, 128, 3,
                                 seed=7, rope_theta=500000.0, plant=0.5),
    # head_dim 64, eight query heads on one KV head, bs 256, top_k 4
    "d64_mqa": synth.Workload("d64_mqa", [777, 1536], 8, 1, 64, 256, 4, seed=8,
                              rope_theta=10000.0),
    # top_k = 1: own block only (block-diagonal causal attention)
    "top1": synth.Workload("top1", [600, 300], 2, 2, 128, 128, 1, seed=9),
    # top_k >= number of blocks: full causal attention
    "full": synth.Workload("full", [640], 4, 1, 128, 128, 16, seed=10),
    # fine blocks, large k
    "fine_k12": synth.Workload("fine_k12", [2053, 900], 4, 4, 128, 128, 12, seed=11,
                               rope_theta=500000.0),
    # uniform batch expressed through cu_seqlens
    "batch3": synth.Workload("batch3", [1024, 1024, 1024], 2, 1, 64, 128, 3, seed=12),
    # odd GQA group (G = 3): own-block tiles pair consecutive query tiles of one head
    "gqa_odd": synth.Workload("gqa_odd", [1500, 640], 6, 2, 128, 256, 3, seed=13,
                              rope_theta=500000.0, plant=0.5),
    # empty sequences inside a packed batch
    "empty_seqs": synth.Workload("empty_seqs", [300, 0, 700, 0, 129], 4, 2, 64, 128, 3, seed=14),
    # the largest block size, one full block plus a partial one
    "bs8192": synth.Workload("bs8192", [9000], 2, 1, 128, 8192, 2, seed=15, rope_theta=500000.0),
    # the largest top_k with more blocks than it
    "top16": synth.Workload("top16", [2560, 1100], 2, 2, 128, 128, 16, seed=16),
    # top_k 6, 8 and 9 (at most 8 past blocks: the gate's two interleaved 8-slot lists), at
    # head_dim 128 and 64
    "k6_d128": synth.Workload("k6_d128", [2000, 1100], 4, 2, 128, 128, 6, seed=18,
                              rope_theta=500000.0, plant=0.5),
    "k8_d64": synth.Workload("k8_d64", [1700, 1300], 4, 1, 64, 128, 8, seed=19,
                             rope_theta=10000.0),
    "k9_d128": synth.Workload("k9_d128", [2300], 2, 2, 128, 128, 9, seed=20),
    # more than 64 past blocks: the gate walks its candidates in several 64-block chunks
    # through the double-buffered score accumulator (73 and 133 blocks)
    "chunks_d128": synth.Workload("chunks_d128", [9300], 4, 2, 128, 128, 3, seed=23,
                                  rope_theta=500000.0, plant=0.5),
    "chunks_d64_k8": synth.Workload("chunks_d64_k8", [17000], 2, 1, 64, 128, 8, seed=24,
                                    rope_theta=500000.0, plant=0.5),
    "chunks_k16": synth.Workload("chunks_k16", [9000, 300], 2, 1, 128, 128, 16, seed=25),
    # the gate's KV-group kernel (exact selection, query heads in groups of four): two head
    # groups per KV head at head_dim 64 (top_k 9), and top_k 16 at head_dim 128, both over
    # more than 64 candidate blocks (several chunks, staged across items)
    "grp_g8_k9_d64": synth.Workload("grp_g8_k9_d64", [9500, 3000], 8, 1, 64, 128, 9, seed=26,
                                    rope_theta=500000.0, plant=0.5),
    "grp_g4_k16": synth.Workload("grp_g4_k16", [12000, 700], 4, 1, 128, 128, 16, seed=27),
    # many short sequences
    "many_seqs": synth.Workload("many_seqs", list(np.random.default_rng(17).integers(1, 300, 300)), 2, 1, 64,
                                128, 3, seed=17),
}


def _inputs(w):
    return w.fill("q"), w.fill("k"), w.fill("v")


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("stages", [False, True])
def test_small_workloads_match_oracle(name, stages, cuda_device):
    w = SMALL[name]
    Q, K, V = _inputs(w)
    gpu = run_gpu(w, Q, K, V, stages=stages)
    orc = oracle.full(problem(w), Q, K, V)
    # pooled keys
    np.testing.assert_allclose(kbar_seq_order(w, gpu["Kbar"]), orc["Kbar"], rtol=0, atol=KBAR_ABS)
    # padded blocks past each sequence's end are zeros
    for s in range(w.num_seqs):
        assert not gpu["Kbar"][s, w.blocks_of(s):].any()
    st = compare(gpu["sel"], gpu["O"], gpu["LSE"], orc)
    assert_parity(st)
    # padding slots are -1 and slot 0 is the own block on every row
    T = w.total_tokens
    for s in range(w.num_seqs):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        own = (np.arange(a, b) - a) // w.block_size
        assert np.all(gpu["sel"][a:b, :, 0] == own[:, None])
    assert gpu["sel"].shape == (T, w.num_q_heads, w.top_k)
