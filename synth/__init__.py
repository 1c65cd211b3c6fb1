"""Seeded synthetic workloads for MoBA causal prefill (input preparation only).

The element values are defined in ``synth.c`` (counter-based splitmix64 words,
Box-Muller normals, optional rotary embedding and planted relevance).  This
module holds no attention arithmetic: the CPU oracle's tests and the GPU path
both consume the buffers it returns, so the two sides see identical inputs.

bf16 tensors are returned as numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, strict fp: no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
            "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Spec(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64),
        ("num_seqs", ctypes.c_int32),
        ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("plant", ctypes.c_double),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.synth_fill.argtypes = [ctypes.POINTER(_Spec), ctypes.c_int, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_rows.argtypes = [ctypes.POINTER(_Spec), ctypes.c_int, i64p, i32p,
                                   ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        lib.synth_rows.restype = ctypes.c_int
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_splitmix64.argtypes = [ctypes.c_uint64]
        lib.synth_splitmix64.restype = ctypes.c_uint64
        lib.synth_plant_target.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int32,
                                           ctypes.c_int, ctypes.c_int]
        lib.synth_plant_target.restype = ctypes.c_int32
        _lib = lib
    return _lib


WHICH = {"q": 0, "k": 1, "v": 2}


@dataclass
class Workload:
    """One MoBA prefill problem: packed sequences, heads, block size, top-k, input recipe."""

    name: str
    seqlens: list
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    seed: int
    rope_theta: float = 0.0
    plant: float = 0.0
    draw_dtype: str = "bf16"  # "f32" for the tiny case, whose draws are fp32
    cu_seqlens: np.ndarray = field(init=False)

    def __post_init__(self):
        self.cu_seqlens = np.zeros(len(self.seqlens) + 1, dtype=np.int32)
        self.cu_seqlens[1:] = np.cumsum(np.asarray(self.seqlens, dtype=np.int64))
        assert int(self.cu_seqlens[-1]) < 2**31

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens)) if self.seqlens else 0

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)

    def blocks_of(self, s: int) -> int:
        return -(-int(self.seqlens[s]) // self.block_size)

    def heads(self, which: str) -> int:
        return self.num_q_heads if which == "q" else self.num_kv_heads

    def _spec(self) -> _Spec:
        sp = _Spec()
        sp.seed = self.seed
        sp.num_seqs = self.num_seqs
        self._cu_keep = np.ascontiguousarray(self.cu_seqlens, dtype=np.int32)
        sp.cu_seqlens = self._cu_keep.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        sp.num_q_heads = self.num_q_heads
        sp.num_kv_heads = self.num_kv_heads
        sp.head_dim = self.head_dim
        sp.block_size = self.block_size
        sp.rope_theta = float(self.rope_theta)
        sp.plant = float(self.plant)
        return sp

    def fill(self, which: str, t0: int = 0, t1: int | None = None, kind: str = "bf16",
             out: np.ndarray | None = None, nthreads: int | None = None) -> np.ndarray:
        """Tensor rows [t0, t1) of Q, K or V as [t1-t0, H, D] (bf16 bits or fp32)."""
        t1 = self.total_tokens if t1 is None else t1
        h = self.heads(which)
        shape = (t1 - t0, h, self.head_dim)
        dt = np.uint16 if kind == "bf16" else np.float32
        if out is None:
            out = np.empty(shape, dtype=dt)
        assert out.dtype == dt and out.shape == shape and out.flags.c_contiguous
        sp = self._spec()
        rc = _load().synth_fill(ctypes.byref(sp), WHICH[which], t0, t1,
                                1 if kind == "bf16" else 0, out.ctypes.data,
                                nthreads or os.cpu_count() or 1)
        if rc:
            raise ValueError("synth_fill failed with code %d" % rc)
        return out

    def rows(self, which: str, tok, head, kind: str = "bf16",
             nthreads: int | None = None) -> np.ndarray:
        """Individual (token, head) rows of Q, K or V as [n, D]."""
        tok = np.ascontiguousarray(tok, dtype=np.int64)
        head = np.ascontiguousarray(head, dtype=np.int32)
        assert tok.shape == head.shape and tok.ndim == 1
        dt = np.uint16 if kind == "bf16" else np.float32
        out = np.empty((tok.size, self.head_dim), dtype=dt)
        sp = self._spec()
        rc = _load().synth_rows(ctypes.byref(sp), WHICH[which],
                                tok.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                head.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                tok.size, 1 if kind == "bf16" else 0, out.ctypes.data,
                                nthreads or os.cpu_count() or 1)
        if rc:
            raise ValueError("synth_rows failed with code %d" % rc)
        return out

    def plant_target(self, s: int, i: int, g: int) -> int:
        return int(_load().synth_plant_target(self.seed, s, i, g, self.num_kv_heads))


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even narrowing of float32 to bf16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def normal(seed: int, tensor_id: int, e: int) -> float:
    return float(_load().synth_normal(seed, tensor_id, e))


def splitmix64(x: int) -> int:
    return int(_load().synth_splitmix64(x & (2**64 - 1)))


# The five workloads: shapes, block sizes, top-k and input recipes of the MoBA
# prefill measurements (tiny fp32 check, 32K MHA, 128K GQA with planted
# relevance, 1M-token GQA with planted relevance, packed varlen with fine blocks).
CONFIGS = {
    "tiny": Workload("tiny", [1024], 1, 1, 64, 128, 3, seed=1001, draw_dtype="f32"),
    "mha32k": Workload("mha32k", [32768], 32, 32, 128, 2048, 3, seed=1002, rope_theta=500000.0),
    "gqa128k": Workload("gqa128k", [131072], 32, 8, 128, 2048, 3, seed=1003,
                        rope_theta=500000.0, plant=0.5),
    "prefill1m": Workload("prefill1m", [1048576], 32, 8, 128, 2048, 3, seed=1004,
                          rope_theta=500000.0, plant=0.5),
    "varlen": Workload("varlen", [131072, 65536, 32768, 16384], 32, 8, 128, 512, 12,
                       seed=1005, rope_theta=500000.0),
}
