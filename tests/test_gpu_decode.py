"""GPU parity of gated decode (moba_decode_fwd) against the fp64 oracle: the new query of a
sequence is its last cached token, so the oracle's row for that token (same gate, same
selection rule, same masked softmax) is the expected result.  Also: decode agrees with the
prefill path's row for the same token, and re-pooling the last block reproduces the full
pooling exactly."""
import numpy as np
import pytest

import oracle
import synth
from _harness import assert_parity, compare, params, problem, run_gpu, to_device_bf16

pytestmark = pytest.mark.gpu

CASES = [
    # lengths 1 (own block only), below, at and past one block, several blocks
    synth.Workload("dec_small", [1, 127, 128, 129, 1000, 2048, 5000], 4, 2, 128, 128, 3, seed=61,
                   rope_theta=500000.0, plant=0.5),
    # head_dim 64, top_k 8, more than 64 candidate blocks (several gate chunks)
    synth.Workload("dec_d64_k8", [3000, 4096, 17000], 8, 2, 64, 128, 8, seed=62, rope_theta=10000.0),
    # top_k 16 with 35 blocks, one KV head for two query heads
    synth.Workload("dec_k16", [9000], 2, 1, 128, 256, 16, seed=63),
    # long caches, Llama-shaped GQA, block 2048
    synth.Workload("dec_long", [40000, 70001, 131072], 32, 8, 128, 2048, 3, seed=64,
                   rope_theta=500000.0, plant=0.5),
    # top_k 1: the own block only
    synth.Workload("dec_top1", [5000, 300, 4097], 4, 4, 128, 512, 1, seed=65),
    # odd group size, block 8192
    synth.Workload("dec_g3_bs8192", [20000, 8192], 6, 2, 128, 8192, 2, seed=66),
    # eight query heads on one KV head with planted relevance: up to eight heads choose the
    # same block, which is read once for each run of four of them
    synth.Workload("dec_mqa8", [5000, 20000, 777], 8, 1, 128, 512, 3, seed=67, rope_theta=500000.0,
                   plant=0.5),
]


def _decode(w, Q, K, V):
    import torch
    import block_sparse_attention_gate_b200 as mb
    p = params(w)
    last = (w.cu_seqlens[1:] - 1).astype(np.int64)
    Qd = to_device_bf16(np.ascontiguousarray(Q[last]))
    Kd, Vd = to_device_bf16(K), to_device_bf16(V)
    kbar = torch.empty(p.kbar_elems, dtype=torch.float32, device="cuda")
    mb.moba_pool_keys(p, Kd, kbar)
    ws = torch.empty(mb.moba_decode_workspace_size(p), dtype=torch.uint8, device="cuda")
    B, hq = w.num_seqs, w.num_q_heads
    sel = torch.full((B, hq, w.top_k), -7, dtype=torch.int32, device="cuda")
    O = torch.full((B, hq, w.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    LSE = torch.full((B, hq), float("nan"), dtype=torch.float32, device="cuda")
    mb.moba_decode_fwd(p, Qd, Kd, Vd, kbar, ws, O, LSE, sel=sel)
    torch.cuda.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    return last, sel.cpu().numpy(), O.float().cpu().numpy(), LSE.cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_matches_oracle(w, cuda_device):
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    last, sel, O, LSE = _decode(w, Q, K, V)
    pr = problem(w)
    kbar = oracle.pool_keys(pr, K)
    hq = w.num_q_heads
    tok = np.repeat(last, hq)
    hd = np.tile(np.arange(hq, dtype=np.int32), last.size)
    orc = oracle.rows(pr, Q[tok, hd], K, V, kbar, tok, hd)
    st = compare(sel.reshape(-1, w.top_k), O.reshape(-1, w.head_dim), LSE.reshape(-1), orc)
    print(w.name, st)
    assert_parity(st, max_excluded_frac=0.02)
    # own block in slot 0, -1 padding after the min(top_k - 1, i) chosen blocks
    own = ((w.cu_seqlens[1:] - w.cu_seqlens[:-1] - 1) // w.block_size)
    assert np.all(sel[:, :, 0] == own[:, None])
    m = np.minimum(w.top_k - 1, own)
    for s in range(w.num_seqs):
        assert np.all(sel[s, :, 1 + m[s]:] == -1)
        assert np.all((sel[s, :, 1:1 + m[s]] >= 0) & (sel[s, :, 1:1 + m[s]] < own[s]))


@pytest.mark.parametrize("w", CASES[:3], ids=lambda w: w.name)
def test_decode_agrees_with_prefill_row(w, cuda_device):
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    last, sel, O, LSE = _decode(w, Q, K, V)
    pre = run_gpu(w, Q, K, V)
    same = np.all(np.sort(sel, axis=-1) == np.sort(pre["sel"][last], axis=-1), axis=-1)
    assert same.mean() >= 0.98
    d = np.abs(O - pre["O"][last])[same]
    assert d.max() <= 1e-2 + 2.0 ** -8 * np.abs(pre["O"][last][same]).max()
    assert np.abs(LSE - pre["LSE"][last])[same].max() <= 1e-3


def test_pool_last_block_reproduces_full_pooling(cuda_device):
    import torch
    import block_sparse_attention_gate_b200 as mb
    w = CASES[0]
    p = params(w)
    Kd = to_device_bf16(w.fill("k"))
    full = torch.empty(p.kbar_elems, dtype=torch.float32, device="cuda")
    mb.moba_pool_keys(p, Kd, full)
    kb = full.view(w.num_seqs, p.max_blocks, w.num_kv_heads, w.head_dim)
    part = kb.clone()
    lastb = [max(0, (int(n) - 1) // w.block_size) for n in w.seqlens]
    for s, b in enumerate(lastb):
        part[s, b] = 12345.0
    mb.moba_pool_last_block(p, Kd, part.view(-1))
    torch.cuda.synchronize()
    assert torch.equal(part, kb)
