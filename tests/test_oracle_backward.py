"""Pins of the fp64 backward oracle (``oracle.backward``) to facts fixed outside it.

- Central finite differences of L = sum(dO * O) through a separately written fp64 forward
  that holds the selection fixed (that forward is itself checked against the forward
  oracle's O first).
- The limits where MoBA is plain causal attention (top_k >= number of blocks) or
  block-diagonal causal attention (top_k = 1): torch autograd through SDPA in fp64.
- Closed-form sums: the rows of P sum to one, so the keys' dV add up to the rows' dO, and
  the rows of dS sum to zero, so the keys' dK add up to zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def _problem(seqlens, hq, hkv, D, bs, k):
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    return oracle.Problem(cu, hq, hkv, D, bs, k, dtype="f32")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _fixed_mask_forward(pr, masks, q, k, v):
    """O of masked softmax attention for fp64 inputs, the keep masks held fixed."""
    T, hq, D = q.shape
    G = hq // k.shape[1]
    scale = 1.0 / math.sqrt(D)
    O = np.zeros((T, hq, D))
    cu = np.asarray(pr.cu_seqlens)
    for s in range(cu.size - 1):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for h in range(hq):
            keep = masks[s][h]
            z = scale * (q[t0:t1, h] @ k[t0:t1, h // G].T)
            z = np.where(keep, z, -np.inf)
            w = np.exp(z - z.max(axis=1, keepdims=True))
            O[t0:t1, h] = (w / w.sum(axis=1, keepdims=True)) @ v[t0:t1, h // G]
    return O


def test_backward_matches_central_finite_differences():
    pr = _problem([40, 24], 2, 1, 4, 8, 2)
    Q, K, V = _rand((64, 2, 4), 1), _rand((64, 1, 4), 2), _rand((64, 1, 4), 3)
    dO = np.random.default_rng(4).standard_normal((64, 2, 4))
    res = ob.backward(pr, Q, K, V, dO)
    masks, fw = ob.keep_masks(pr, Q, K, V)
    q, k, v = (x.astype(np.float64) for x in (Q, K, V))
    # the separately written forward reproduces the forward oracle under its selection
    np.testing.assert_allclose(_fixed_mask_forward(pr, masks, q, k, v), fw["O"], rtol=0, atol=1e-13)

    def loss(qq, kk, vv):
        return float(np.sum(dO * _fixed_mask_forward(pr, masks, qq, kk, vv)))

    rng = np.random.default_rng(5)
    eps = 1e-6
    for name, base, grad in (("Q", q, res["dQ"]), ("K", k, res["dK"]), ("V", v, res["dV"])):
        for _ in range(16):
            idx = tuple(int(rng.integers(0, n)) for n in base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"Q": q, "K": k, "V": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (loss(args_p["Q"], args_p["K"], args_p["V"]) - loss(args_m["Q"], args_m["K"], args_m["V"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 + 1e-6 * abs(fd), (name, idx, fd, grad[idx])


def _autograd_reference(Q, K, V, dO, mask):
    T, hq, D = Q.shape
    G = hq // K.shape[1]
    q = torch.tensor(Q.astype(np.float64)).permute(1, 0, 2).requires_grad_()
    k = torch.tensor(K.astype(np.float64)).permute(1, 0, 2).requires_grad_()
    v = torch.tensor(V.astype(np.float64)).permute(1, 0, 2).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, 0), v.repeat_interleave(G, 0), attn_mask=torch.from_numpy(mask))
    (o * torch.tensor(dO).permute(1, 0, 2)).sum().backward()
    return [x.grad.permute(1, 0, 2).numpy() for x in (q, k, v)]


@pytest.mark.parametrize("S,bs,k", [(50, 16, 10), (64, 64, 3)])
def test_full_attention_limit_matches_autograd(S, bs, k):
    pr = _problem([S], 4, 2, 8, bs, k)
    Q, K, V = _rand((S, 4, 8), 11), _rand((S, 2, 8), 12), _rand((S, 2, 8), 13)
    dO = np.random.default_rng(14).standard_normal((S, 4, 8))
    res = ob.backward(pr, Q, K, V, dO)
    mask = np.tril(np.ones((S, S), dtype=bool))
    dq, dk, dv = _autograd_reference(Q, K, V, dO, mask)
    for got, want in ((res["dQ"], dq), (res["dK"], dk), (res["dV"], dv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_top1_block_diagonal_matches_autograd():
    S, bs = 72, 16
    pr = _problem([S], 2, 1, 8, bs, 1)
    Q, K, V = _rand((S, 2, 8), 21), _rand((S, 1, 8), 22), _rand((S, 1, 8), 23)
    dO = np.random.default_rng(24).standard_normal((S, 2, 8))
    res = ob.backward(pr, Q, K, V, dO)
    t = np.arange(S)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] // bs == t[:, None] // bs)
    dq, dk, dv = _autograd_reference(Q, K, V, dO, mask)
    for got, want in ((res["dQ"], dq), (res["dK"], dk), (res["dV"], dv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_sparse_backward_closed_form_sums():
    seqlens = [96, 40]
    pr = _problem(seqlens, 4, 2, 8, 8, 3)
    T = sum(seqlens)
    Q, K, V = _rand((T, 4, 8), 31), _rand((T, 2, 8), 32), _rand((T, 2, 8), 33)
    dO = np.random.default_rng(34).standard_normal((T, 4, 8))
    res = ob.backward(pr, Q, K, V, dO)
    cu = np.asarray(pr.cu_seqlens)
    for s in range(len(seqlens)):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for g in range(2):
            heads = [2 * g, 2 * g + 1]
            np.testing.assert_allclose(res["dV"][t0:t1, g].sum(0), dO[t0:t1, heads].sum((0, 1)), rtol=0, atol=1e-11)
            np.testing.assert_allclose(res["dK"][t0:t1, g].sum(0), 0.0, rtol=0, atol=1e-11)
    # the selection is the forward's: own block always kept, nothing from a later block
    assert np.all(res["sel"][:, :, 0] == (np.concatenate([np.arange(n) for n in seqlens]) // 8)[:, None])
