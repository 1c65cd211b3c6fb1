"""moba_gate_topk_noalloc, the gate entry point for callers that cannot allocate device
memory (graph capture, allocation-free serving runtimes, raw-pointer host programs): called
through the C ABI twice in a row on different problems, each result must equal what the
workspace-taking moba_gate_topk returns for the same inputs (integer output: exact)."""
import ctypes

import numpy as np
import pytest

import synth
from _harness import params, to_device_bf16

pytestmark = pytest.mark.gpu

CASES = [
    synth.Workload("na_a", [1000, 333, 2125, 128, 1], 4, 2, 128, 128, 3, seed=21,
                   rope_theta=500000.0, plant=0.5),
    synth.Workload("na_b", [4096, 777], 8, 2, 64, 256, 6, seed=22, rope_theta=10000.0),
]


def _gate_both(w):
    import torch
    import block_sparse_attention_gate_b200 as mb
    lib = mb.load()
    p = params(w)
    Q, K = to_device_bf16(w.fill("q")), to_device_bf16(w.fill("k"))
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device="cuda")
    mb.moba_pool_keys(p, K, kbar)
    ws = mb.alloc_workspace(p)
    T = w.total_tokens
    ref = torch.full((T, w.num_q_heads, w.top_k), -7, dtype=torch.int32, device="cuda")
    got = torch.full_like(ref, -9)
    mb.moba_gate_topk(p, Q, kbar, ref, ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moba_gate_topk_noalloc(p.ref(), Q.data_ptr(), kbar.data_ptr(), got.data_ptr(), stream)
    assert rc == 0, lib.moba_last_error()
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    return ref.cpu().numpy(), got.cpu().numpy()


def test_noalloc_gate_matches_workspace_gate_twice():
    for w in CASES:  # two calls in a row share the library's scratch array
        ref, got = _gate_both(w)
        np.testing.assert_array_equal(got, ref)


def test_noalloc_gate_rejects_problems_beyond_its_scratch():
    import block_sparse_attention_gate_b200 as mb
    lib = mb.load()
    # 64 sequences x 1024 blocks x 8 KV heads x 128 dims = 2^26 > 2^21 elements
    p = mb.MobaParams(None, 32, 8, 128, 128, 3, num_seqs=64, max_seqlen=128 * 1024)
    rc = lib.moba_gate_topk_noalloc(p.ref(), 256, 256, 256, None)
    assert rc == 2
    assert b"scratch" in lib.moba_last_error()
