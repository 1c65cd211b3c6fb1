"""fp64 CPU oracle for the MoBA backward pass -- TEST INFRASTRUCTURE ONLY.

MoBA is trained (MoBA README, bullet "Trainable Block Sparse Attention"; youleyou.com,
"Kimi发布MoBA突破性实现无限上下文": the model is trained with the block attention in
place), and its gate has no parameters (MoBA README, "Parameter-less Gating Mechanism"):
the top-k selection is piecewise constant in the inputs, so gradients flow only through
the attention over the selected blocks, with the selection held fixed.

The backward pass is therefore the gradient of masked softmax attention under MoBA's
mask: for a query row p with keep[p, j] (key j in a selected block and j <= p),

    P[p, j]  = keep[p, j] * exp(scale <Q_p, K_j> - LSE_p)
    dV_j    += sum_p P[p, j] dO_p
    dP[p, j] = <dO_p, V_j>
    D_p      = <dO_p, O_p>              (= sum_j P[p, j] dP[p, j])
    dS[p, j] = P[p, j] (dP[p, j] - D_p)
    dQ_p     = scale sum_j dS[p, j] K_j
    dK_j    += scale sum_p dS[p, j] Q_p

summed over the query heads of a KV head's group for dK and dV.  The selection, O and
LSE come from the forward oracle (``oracle.rows`` with the materialised block mask).
Dense per-sequence matrices in numpy fp64: meant for test sizes (a few thousand tokens).
"""
from __future__ import annotations

import numpy as np

from . import Problem, pool_keys, rows


def widen(pr: Problem, a: np.ndarray) -> np.ndarray:
    """Inputs as the oracle reads them (bf16 bit patterns or fp32), widened to fp64."""
    a = pr._in(a)
    if pr.dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def keep_masks(pr: Problem, Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> tuple[list, dict]:
    """Per sequence, the boolean key masks [Hq, L, L] of the forward's selection, plus the
    forward outputs (O, lse in fp64, shaped [T, Hq, ...])."""
    T, hq, D = Q.shape
    tt, hh = np.meshgrid(np.arange(T, dtype=np.int64), np.arange(hq, dtype=np.int32), indexing="ij")
    Kbar = pool_keys(pr, K)
    fw = rows(pr, Q.reshape(T * hq, D), K, V, Kbar, tt.ravel(), hh.ravel(), mask=True)
    blocks = fw["mask"].reshape(T, hq, -1).astype(bool)
    cu = np.asarray(pr.cu_seqlens, dtype=np.int64)
    bs = pr.block_size
    masks = []
    for s in range(cu.size - 1):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        L = t1 - t0
        pos = np.arange(L)
        causal = pos[None, :] <= pos[:, None]
        m = np.empty((hq, L, L), dtype=bool)
        for h in range(hq):
            m[h] = blocks[t0:t1, h][:, pos // bs] & causal
        masks.append(m)
    out = {"O": fw["O"].reshape(T, hq, D), "lse": fw["lse"].reshape(T, hq), "sel": fw["sel"].reshape(T, hq, -1)}
    return masks, out


def backward(pr: Problem, Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray) -> dict:
    """dQ [T, Hq, D], dK and dV [T, Hkv, D] (fp64) of MoBA attention for the upstream
    gradient dO [T, Hq, D]; also returns the forward's O, lse and sel."""
    T, hq, D = Q.shape
    hkv = K.shape[1]
    G = hq // hkv
    scale = pr.softmax_scale if pr.softmax_scale > 0 else 1.0 / np.sqrt(D)
    masks, fw = keep_masks(pr, Q, K, V)
    q, k, v = widen(pr, Q), widen(pr, K), widen(pr, V)
    dO = np.asarray(dO, dtype=np.float64)
    dQ = np.zeros((T, hq, D))
    dK = np.zeros((T, hkv, D))
    dV = np.zeros((T, hkv, D))
    cu = np.asarray(pr.cu_seqlens, dtype=np.int64)
    for s in range(cu.size - 1):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        if t1 == t0:
            continue
        for h in range(hq):
            g = h // G
            keep = masks[s][h]
            z = scale * (q[t0:t1, h] @ k[t0:t1, g].T)
            P = np.where(keep, np.exp(np.where(keep, z, 0.0) - fw["lse"][t0:t1, h][:, None]), 0.0)
            do = dO[t0:t1, h]
            dV[t0:t1, g] += P.T @ do
            dP = do @ v[t0:t1, g].T
            Dp = np.sum(do * fw["O"][t0:t1, h], axis=1)
            dS = P * (dP - Dp[:, None])
            dQ[t0:t1, h] = scale * (dS @ k[t0:t1, g])
            dK[t0:t1, g] += scale * (dS.T @ q[t0:t1, h])
    return {"dQ": dQ, "dK": dK, "dV": dV, **fw}
