"""CPU fp64 oracle for MoBA causal prefill -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The GPU library
never loads it and shares no code with it.

The arithmetic lives in ``moba_oracle.c`` (mask-based form: pool, score, select,
materialise the block mask, masked softmax; every step in fp64).  This module
only compiles it with gcc and marshals numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py`` against brute
force, closed forms, invariants and a library attention routine; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moba_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into liboracle.so next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
            "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
        ("dtype", ctypes.c_int32),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        vp = ctypes.c_void_p
        lib.oracle_block_offsets.argtypes = [P, vp]
        lib.oracle_block_offsets.restype = ctypes.c_int64
        lib.oracle_pool_keys.argtypes = [P, vp, vp, ctypes.c_int]
        lib.oracle_pool_keys.restype = ctypes.c_int
        lib.oracle_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.c_int64,
                                    vp, vp, vp, vp, vp, vp, ctypes.c_int]
        lib.oracle_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


@dataclass
class Problem:
    """Shapes and hyper-parameters of one packed MoBA prefill problem."""

    cu_seqlens: np.ndarray
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    softmax_scale: float = 0.0
    dtype: str = "bf16"  # "bf16" (uint16 bit patterns) or "f32"

    def _c(self) -> _Problem:
        self._cu = np.ascontiguousarray(self.cu_seqlens, dtype=np.int32)
        p = _Problem()
        p.num_seqs = self._cu.size - 1
        p.cu_seqlens = self._cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        p.num_q_heads = self.num_q_heads
        p.num_kv_heads = self.num_kv_heads
        p.head_dim = self.head_dim
        p.block_size = self.block_size
        p.top_k = self.top_k
        p.softmax_scale = self.softmax_scale
        p.dtype = 1 if self.dtype == "bf16" else 0
        return p

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    def block_offsets(self) -> np.ndarray:
        off = np.zeros(len(self.cu_seqlens), dtype=np.int64)
        p = self._c()
        nb = _load().oracle_block_offsets(ctypes.byref(p), off.ctypes.data)
        if nb < 0:
            raise ValueError("invalid problem")
        return off

    def _in(self, a: np.ndarray) -> np.ndarray:
        want = np.uint16 if self.dtype == "bf16" else np.float32
        a = np.ascontiguousarray(a)
        if a.dtype != want:
            raise TypeError("expected %s input, got %s" % (want, a.dtype))
        return a


def _threads(n):
    return n or os.cpu_count() or 1


def pool_keys(pr: Problem, K: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Block means of K: [NB, Hkv, D] float64, blocks in sequence order."""
    K = pr._in(K)
    nb = int(pr.block_offsets()[-1])
    out = np.empty((nb, pr.num_kv_heads, pr.head_dim), dtype=np.float64)
    p = pr._c()
    rc = _load().oracle_pool_keys(ctypes.byref(p), K.ctypes.data, out.ctypes.data,
                                  _threads(nthreads))
    if rc:
        raise ValueError("oracle_pool_keys failed (%d)" % rc)
    return out


def rows(pr: Problem, Qrows: np.ndarray, K: np.ndarray | None, V: np.ndarray | None,
         Kbar: np.ndarray, row_t, row_h, attention: bool = True, mask: bool = False,
         nthreads: int | None = None) -> dict:
    """Oracle outputs for query rows (row_t[r], row_h[r]); Qrows [n, D] holds their queries.

    Returns a dict with sel [n, top_k] int32, gap [n], gmax [n] and, when
    ``attention`` is set, O [n, D] and lse [n] (fp64); ``mask`` adds the
    materialised block mask [n, max_blocks] (uint8).
    """
    Qrows = pr._in(Qrows)
    row_t = np.ascontiguousarray(row_t, dtype=np.int64)
    row_h = np.ascontiguousarray(row_h, dtype=np.int32)
    n = row_t.size
    assert Qrows.shape == (n, pr.head_dim)
    Kbar = np.ascontiguousarray(Kbar, dtype=np.float64)
    out = {
        "sel": np.empty((n, pr.top_k), dtype=np.int32),
        "gap": np.empty(n, dtype=np.float64),
        "gmax": np.empty(n, dtype=np.float64),
    }
    kp = vp = None
    if attention:
        K = pr._in(K)
        V = pr._in(V)
        kp, vp = K.ctypes.data, V.ctypes.data
        out["O"] = np.empty((n, pr.head_dim), dtype=np.float64)
        out["lse"] = np.empty(n, dtype=np.float64)
    if mask:
        off = pr.block_offsets()
        mb = int(np.max(np.diff(off))) if off.size > 1 else 0
        out["mask"] = np.empty((n, mb), dtype=np.uint8)
    p = pr._c()
    rc = _load().oracle_rows(
        ctypes.byref(p), Qrows.ctypes.data, kp, vp, Kbar.ctypes.data,
        row_t.ctypes.data, row_h.ctypes.data, n,
        out["sel"].ctypes.data, out["gap"].ctypes.data, out["gmax"].ctypes.data,
        out["O"].ctypes.data if attention else None,
        out["lse"].ctypes.data if attention else None,
        out["mask"].ctypes.data if mask else None, _threads(nthreads))
    if rc:
        raise ValueError("oracle_rows failed (%d)" % rc)
    return out


def full(pr: Problem, Q: np.ndarray, K: np.ndarray, V: np.ndarray,
         nthreads: int | None = None) -> dict:
    """Oracle over every (token, query head) row; outputs reshaped to [T, Hq, ...]."""
    T, hq, D = Q.shape
    tt, hh = np.meshgrid(np.arange(T, dtype=np.int64), np.arange(hq, dtype=np.int32),
                         indexing="ij")
    Kbar = pool_keys(pr, K, nthreads)
    r = rows(pr, Q.reshape(T * hq, D), K, V, Kbar, tt.ravel(), hh.ravel(), nthreads=nthreads)
    return {
        "Kbar": Kbar,
        "sel": r["sel"].reshape(T, hq, pr.top_k),
        "gap": r["gap"].reshape(T, hq),
        "gmax": r["gmax"].reshape(T, hq),
        "O": r["O"].reshape(T, hq, D),
        "lse": r["lse"].reshape(T, hq),
    }
