"""Pins of the fp64 CPU oracle to facts fixed outside it.

The pages print no worked numeric example, so each oracle step is pinned by
something independent of its own code: closed forms, brute-force enumeration
on tiny inputs, a library attention routine (torch SDPA in fp64) in the limits
where MoBA reduces to plain causal or block-diagonal attention, and invariants
that the method states (own block always chosen, no future key weighted,
exactly min(top_k, i+1) blocks per row).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _problem(seqlens, hq, hkv, D, bs, k, dtype="f32"):
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    return oracle.Problem(cu, hq, hkv, D, bs, k, dtype=dtype)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _all_rows(pr, Q, K, V, **kw):
    return oracle.full(pr, Q, K, V, **kw)


# ------------------------------------------------------------------ pooling
def test_pool_constant_blocks_give_the_constant():
    # keys constant inside each block (ragged last block included): the mean is that constant
    seqlens = [37, 16, 5]
    pr = _problem(seqlens, 2, 2, 8, 8, 3)
    T = sum(seqlens)
    K = np.empty((T, 2, 8), dtype=np.float32)
    want = []
    for s, L in enumerate(seqlens):
        t0 = int(pr.cu_seqlens[s])
        for b in range(-(-L // 8)):
            c = np.float32(0.25 * (s + 1) - 0.125 * b) + np.arange(16, dtype=np.float32).reshape(2, 8)
            K[t0 + 8 * b: t0 + min(L, 8 * b + 8)] = c
            want.append(c)
    got = oracle.pool_keys(pr, K)
    assert got.shape == (len(want), 2, 8)
    np.testing.assert_array_equal(got, np.stack(want).astype(np.float64))


def test_pool_is_the_block_mean_over_valid_tokens():
    seqlens = [29, 3]
    pr = _problem(seqlens, 3, 3, 4, 8, 2)
    K = _rand((32, 3, 4), 1)
    got = oracle.pool_keys(pr, K)
    # independent: math.fsum of each block's exact values divided by its valid-token count
    blocks = [(0, 8), (8, 16), (16, 24), (24, 29), (29, 32)]
    for gb, (a, b) in enumerate(blocks):
        for g in range(3):
            for d in range(4):
                ref = math.fsum(float(K[t, g, d]) for t in range(a, b)) / (b - a)
                assert abs(got[gb, g, d] - ref) <= 1e-15 * max(1.0, abs(ref))


# -------------------------------------------------------------- gate + top-k
def _brute_selection(q, kbar_blocks, i, k):
    """Enumerate every subset of size m of the past blocks; keep the best one.

    The best subset maximises its scores sorted in descending order
    (lexicographically); among equal score vectors the lower indices win.
    """
    scores = [math.fsum(float(a) * float(b) for a, b in zip(q, kb)) for kb in kbar_blocks[:i]]
    m = min(k - 1, i)
    best = None
    for sub in itertools.combinations(range(i), m):
        key = (tuple(sorted((scores[b] for b in sub), reverse=True)), tuple(-b for b in sorted(sub)))
        if best is None or key > best[0]:
            best = (key, sub)
    chosen = sorted(best[1], key=lambda b: (-scores[b], b))
    return [i] + chosen + [-1] * (k - 1 - m)


@pytest.mark.parametrize("bs,k,seed", [(4, 1, 0), (4, 2, 1), (8, 3, 2), (4, 5, 3), (8, 5, 4), (4, 3, 5)])
def test_gate_matches_bruteforce_enumeration(bs, k, seed):
    S, D, hq, hkv = 48, 6, 2, 1
    pr = _problem([S], hq, hkv, D, bs, k)
    Q, K, V = _rand((S, hq, D), seed), _rand((S, hkv, D), seed + 100), _rand((S, hkv, D), seed + 200)
    out = _all_rows(pr, Q, K, V)
    nb = -(-S // bs)
    kbar = [[math.fsum(float(K[t, 0, d]) for t in range(b * bs, min(S, b * bs + bs))) /
             (min(S, b * bs + bs) - b * bs) for d in range(D)] for b in range(nb)]
    for t in range(S):
        for h in range(hq):
            want = _brute_selection(Q[t, h], kbar, t // bs, k)
            assert list(out["sel"][t, h]) == want, (t, h)


def test_gate_ties_go_to_the_lower_block_index():
    # blocks 0, 2 and 3 share the same mean key; block 1 is worse; query positive
    bs, D = 4, 3
    S = 6 * bs
    pr = _problem([S], 1, 1, D, bs, 3)
    K = np.zeros((S, 1, D), dtype=np.float32)
    for b, v in enumerate([1.0, 0.5, 1.0, 1.0, 0.0, 0.0]):
        K[b * bs:(b + 1) * bs] = v
    Q = np.ones((S, 1, D), dtype=np.float32)
    V = _rand((S, 1, D), 3)
    out = _all_rows(pr, Q, K, V)
    # a query in block 4 sees candidates 0..3 with scores 3, 1.5, 3, 3 -> picks 0 then 2
    for t in range(4 * bs, 5 * bs):
        assert list(out["sel"][t, 0]) == [4, 0, 2]
    # a query in block 5 sees 0..4 (block 4 scores 0) -> still 0 then 2
    for t in range(5 * bs, 6 * bs):
        assert list(out["sel"][t, 0]) == [5, 0, 2]
    # block 3 queries: candidates 0..2 -> 0, 2
    for t in range(3 * bs, 4 * bs):
        assert list(out["sel"][t, 0]) == [3, 0, 2]


def test_gate_selection_invariant_under_positive_key_scaling():
    pr = _problem([64], 2, 1, 8, 8, 3)
    Q, K, V = _rand((64, 2, 8), 7), _rand((64, 1, 8), 8), _rand((64, 1, 8), 9)
    a = _all_rows(pr, Q, K, V)["sel"]
    b = _all_rows(pr, Q, (2.0 * K).astype(np.float32), V)["sel"]
    np.testing.assert_array_equal(a, b)


def test_gap_and_gmax_definitions():
    pr = _problem([40], 1, 1, 4, 4, 3)
    Q, K, V = _rand((40, 1, 4), 11), _rand((40, 1, 4), 12), _rand((40, 1, 4), 13)
    out = _all_rows(pr, Q, K, V)
    kb = out["Kbar"]
    for t in range(40):
        i = t // 4
        sc = [float(np.dot(Q[t, 0].astype(np.float64), kb[b, 0])) for b in range(i)]
        if i <= 2:
            assert math.isinf(out["gap"][t, 0])
        else:
            srt = sorted(sc, reverse=True)
            assert abs(out["gap"][t, 0] - (srt[1] - srt[2])) < 1e-12
        assert abs(out["gmax"][t, 0] - (max(map(abs, sc)) if sc else 0.0)) < 1e-12


# ------------------------------------------------- attention: library limits
def _sdpa(Q, K, V, mask=None, causal=False):
    """torch SDPA in fp64 on [T,H,D] inputs (GQA by repeating KV heads) plus a logsumexp."""
    T, hq, D = Q.shape
    G = hq // K.shape[1]
    q = torch.from_numpy(Q.astype(np.float64)).permute(1, 0, 2)
    k = torch.from_numpy(K.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    v = torch.from_numpy(V.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    if causal:
        m = torch.ones(T, T, dtype=torch.bool).tril()
    else:
        m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)
    z = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    lse = torch.logsumexp(z.masked_fill(~m, float("-inf")), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


@pytest.mark.parametrize("seqlens,bs,k", [([200], 16, 13), ([200], 16, 40), ([97], 128, 3), ([64], 64, 1)])
def test_full_attention_limit(seqlens, bs, k):
    # top_k >= number of blocks, or block_size >= S: MoBA is plain causal attention
    S = seqlens[0]
    pr = _problem(seqlens, 4, 2, 16, bs, k)
    Q, K, V = _rand((S, 4, 16), 21), _rand((S, 2, 16), 22), _rand((S, 2, 16), 23)
    out = _all_rows(pr, Q, K, V)
    o_ref, lse_ref = _sdpa(Q, K, V, causal=True)
    np.testing.assert_allclose(out["O"], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse_ref, rtol=0, atol=1e-12)


def test_top1_is_block_diagonal_causal_attention():
    S, bs = 150, 32
    pr = _problem([S], 2, 1, 8, bs, 1)
    Q, K, V = _rand((S, 2, 8), 31), _rand((S, 1, 8), 32), _rand((S, 1, 8), 33)
    out = _all_rows(pr, Q, K, V)
    t = np.arange(S)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] // bs == t[:, None] // bs)
    o_ref, lse_ref = _sdpa(Q, K, V, mask=mask)
    np.testing.assert_allclose(out["O"], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse_ref, rtol=0, atol=1e-12)


def test_sparse_rows_match_sdpa_with_the_oracle_mask():
    # general top-k: SDPA under the block mask built from the brute-force selection
    S, bs, k, D = 96, 8, 3, 8
    pr = _problem([S], 1, 1, D, bs, k)
    Q, K, V = _rand((S, 1, D), 41), _rand((S, 1, D), 42), _rand((S, 1, D), 43)
    out = _all_rows(pr, Q, K, V)
    nb = S // bs
    kbar = [[float(np.mean(K[b * bs:(b + 1) * bs, 0, d].astype(np.float64))) for d in range(D)]
            for b in range(nb)]
    mask = np.zeros((S, S), dtype=bool)
    for t in range(S):
        for b in _brute_selection(Q[t, 0], kbar, t // bs, k):
            if b >= 0:
                mask[t, b * bs:(b + 1) * bs] = True
        mask[t, t + 1:] = False
    o_ref, lse_ref = _sdpa(Q, K, V, mask=mask)
    np.testing.assert_allclose(out["O"], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse_ref, rtol=0, atol=1e-12)


def test_bruteforce_attention_loops():
    S, bs, k, D = 24, 4, 2, 3
    pr = _problem([S], 1, 1, D, bs, k)
    Q, K, V = _rand((S, 1, D), 51), _rand((S, 1, D), 52), _rand((S, 1, D), 53)
    out = _all_rows(pr, Q, K, V)
    kbar = [[math.fsum(float(K[t, 0, d]) for t in range(b * bs, b * bs + bs)) / bs for d in range(D)]
            for b in range(S // bs)]
    for t in range(S):
        blocks = [b for b in _brute_selection(Q[t, 0], kbar, t // bs, k) if b >= 0]
        keys = [j for b in blocks for j in range(b * bs, b * bs + bs) if j <= t]
        z = [sum(float(Q[t, 0, d]) * float(K[j, 0, d]) for d in range(D)) / math.sqrt(D) for j in keys]
        zm = max(z)
        ssum = math.fsum(math.exp(x - zm) for x in z)
        lse = zm + math.log(ssum)
        o = [math.fsum(math.exp(zj - lse) * float(V[j, 0, d]) for zj, j in zip(z, keys)) for d in range(D)]
        assert abs(out["lse"][t, 0] - lse) < 1e-12
        np.testing.assert_allclose(out["O"][t, 0], o, rtol=0, atol=1e-12)


# ----------------------------------------------------------------- invariants
def test_invariants_onehot_value_probe():
    # V = one-hot(key position): O exposes the attention weights of every key
    S, bs, k = 64, 8, 3
    pr = _problem([S], 2, 1, S, bs, k)
    Q, K = _rand((S, 2, S), 61), _rand((S, 1, S), 62)
    V = np.eye(S, dtype=np.float32).reshape(S, 1, S)
    out = _all_rows(pr, Q, K, V, )
    mask = oracle.rows(pr, Q.reshape(-1, S), K, V, out["Kbar"],
                       np.repeat(np.arange(S), 2), np.tile(np.arange(2), S), attention=False,
                       mask=True)["mask"].reshape(S, 2, -1)
    for t in range(S):
        i = t // bs
        for h in range(2):
            w = out["O"][t, h]
            sel = out["sel"][t, h]
            assert sel[0] == i                                   # own block always chosen
            assert (sel >= 0).sum() == min(k, i + 1)             # exactly min(k, i+1) blocks
            assert np.all(w[t + 1:] == 0.0)                      # no future key weighted
            chosen = set(int(b) for b in sel if b >= 0)
            for j in range(t + 1):
                assert (w[j] > 0) == ((j // bs) in chosen)       # weight only on chosen blocks
            assert abs(w.sum() - 1.0) < 1e-12                    # weights sum to one
            assert mask[t, h].sum() == min(k, i + 1) and mask[t, h, i] == 1
            assert not mask[t, h, i + 1:].any()


def test_invariants_constant_values_and_lse_bound():
    S, bs, k, D = 80, 16, 2, 8
    pr = _problem([S], 1, 1, D, bs, k)
    Q, K = _rand((S, 1, D), 71), _rand((S, 1, D), 72)
    V = np.ones((S, 1, D), dtype=np.float32)
    out = _all_rows(pr, Q, K, V)
    np.testing.assert_allclose(out["O"], 1.0, rtol=0, atol=1e-13)
    for t in range(S):
        zmax = max(float(np.dot(Q[t, 0].astype(np.float64), K[j, 0].astype(np.float64))) / math.sqrt(D)
                   for j in range(t + 1) if (j // bs) in set(out["sel"][t, 0]))
        assert out["lse"][t, 0] >= zmax - 1e-12
    # the first token attends to itself only: LSE = its own logit, O = its own value
    assert abs(out["lse"][0, 0] - float(np.dot(Q[0, 0].astype(np.float64), K[0, 0])) / math.sqrt(D)) < 1e-12


def test_packed_sequences_are_independent():
    seqlens = [40, 17, 64]
    pr = _problem(seqlens, 2, 1, 8, 8, 3)
    T = sum(seqlens)
    Q, K, V = _rand((T, 2, 8), 81), _rand((T, 1, 8), 82), _rand((T, 1, 8), 83)
    packed = _all_rows(pr, Q, K, V)
    t0 = 0
    for L in seqlens:
        one = _all_rows(_problem([L], 2, 1, 8, 8, 3), Q[t0:t0 + L], K[t0:t0 + L], V[t0:t0 + L])
        np.testing.assert_array_equal(packed["sel"][t0:t0 + L], one["sel"])
        np.testing.assert_array_equal(packed["O"][t0:t0 + L], one["O"])
        np.testing.assert_array_equal(packed["lse"][t0:t0 + L], one["lse"])
        t0 += L


def test_gqa_equals_mha_with_repeated_kv_heads():
    S = 72
    Q, K, V = _rand((S, 4, 8), 91), _rand((S, 2, 8), 92), _rand((S, 2, 8), 93)
    gqa = _all_rows(_problem([S], 4, 2, 8, 8, 3), Q, K, V)
    Kr = torch.from_numpy(K).repeat_interleave(2, dim=1).numpy()
    Vr = torch.from_numpy(V).repeat_interleave(2, dim=1).numpy()
    mha = _all_rows(_problem([S], 4, 4, 8, 8, 3), Q, Kr, Vr)
    np.testing.assert_array_equal(gqa["sel"], mha["sel"])
    np.testing.assert_array_equal(gqa["O"], mha["O"])


def test_bf16_inputs_widen_exactly():
    S = 32
    pr32 = _problem([S], 1, 1, 8, 8, 2, dtype="f32")
    prb = _problem([S], 1, 1, 8, 8, 2, dtype="bf16")
    Q, K, V = _rand((S, 1, 8), 101), _rand((S, 1, 8), 102), _rand((S, 1, 8), 103)
    Qb, Kb, Vb = (synth.f32_to_bf16_bits(x) for x in (Q, K, V))
    a = _all_rows(prb, Qb, Kb, Vb)
    b = _all_rows(pr32, synth.bf16_bits_to_f32(Qb), synth.bf16_bits_to_f32(Kb), synth.bf16_bits_to_f32(Vb))
    np.testing.assert_array_equal(a["O"], b["O"])
    np.testing.assert_array_equal(a["sel"], b["sel"])


def test_sampled_rows_equal_full_rows():
    w = synth.Workload("t", [300, 133], 4, 2, 16, 32, 3, seed=5, rope_theta=10000.0, plant=0.5)
    pr = oracle.Problem(w.cu_seqlens, 4, 2, 16, 32, 3, dtype="bf16")
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    full = oracle.full(pr, Q, K, V)
    tok = np.array([0, 31, 32, 299, 300, 432])
    hd = np.array([0, 1, 2, 3, 0, 3])
    r = oracle.rows(pr, w.rows("q", tok, hd), K, V, full["Kbar"], tok, hd)
    np.testing.assert_array_equal(r["sel"], full["sel"][tok, hd])
    np.testing.assert_array_equal(r["O"], full["O"][tok, hd])


def test_bf16_ulp_helper_of_the_parity_rule():
    from _harness import bf16_ulp
    np.testing.assert_array_equal(bf16_ulp(np.array([1.0, 1.5, 2.0, 4.5, -0.3])),
                                  [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -5, 2.0 ** -9])
