"""MoBA (Mixture of Block Attention) causal prefill on B200: Python binding of libmoba.so.

The binding only marshals arguments: every step of the forward pass runs in the
library's sm_100a kernels.  PyTorch provides device memory and streams.  There is
no fallback: if the CUDA library is missing, every call raises.

C-ABI entry points (same names here): ``moba_pool_keys``, ``moba_gate_topk``,
``moba_attn_fwd``, ``moba_fwd``, ``moba_workspace_size``, ``moba_kbar_elems``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoba.so")
_lib = None

STATUS = {0: "MOBA_OK", 1: "MOBA_ERR_INVALID_ARG", 2: "MOBA_ERR_UNSUPPORTED",
          3: "MOBA_ERR_ALIGNMENT", 4: "MOBA_ERR_WORKSPACE", 5: "MOBA_ERR_CUDA",
          6: "MOBA_ERR_DEVICE"}

EXPORTS = ("moba_kbar_elems", "moba_workspace_size", "moba_pool_keys", "moba_gate_topk",
           "moba_attn_fwd", "moba_fwd", "moba_route", "moba_attn_past", "moba_attn_self_merge",
           "moba_launches_per_forward", "moba_read_device_error", "moba_status_string",
           "moba_last_error", "moba_gate_topk_noalloc", "moba_selftest_bounded_wait",
           "moba_host_staging_size", "moba_fwd_host", "moba_attn_naive", "moba_decode_workspace_size",
           "moba_decode_fwd", "moba_pool_last_block", "moba_bwd_workspace_size", "moba_attn_bwd")


class MobaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), detail))
        self.status = status


class _CParams(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("cu_seqlens_host", ctypes.POINTER(ctypes.c_int32)),
        ("cu_seqlens", ctypes.c_void_p),
        ("max_seqlen", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
    ]


def load():
    """Load libmoba.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoba.so is not built (%s); run block_sparse_attention_gate_b200/build.py"
                               % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(_CParams)
        vp = ctypes.c_void_p
        sz = ctypes.c_size_t
        lib.moba_kbar_elems.argtypes = [P]
        lib.moba_kbar_elems.restype = sz
        lib.moba_workspace_size.argtypes = [P]
        lib.moba_workspace_size.restype = sz
        lib.moba_pool_keys.argtypes = [P, vp, vp, vp]
        lib.moba_gate_topk.argtypes = [P, vp, vp, vp, vp, sz, vp]
        lib.moba_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, sz, vp, vp, vp]
        lib.moba_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp]
        lib.moba_route.argtypes = [P, vp, vp, sz, vp]
        lib.moba_attn_past.argtypes = [P, vp, vp, vp, vp, sz, vp]
        lib.moba_attn_self_merge.argtypes = [P, vp, vp, vp, vp, vp, sz, vp, vp, vp]
        lib.moba_bwd_workspace_size.argtypes = [P]
        lib.moba_bwd_workspace_size.restype = sz
        lib.moba_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp, vp]
        lib.moba_attn_bwd.restype = ctypes.c_int
        lib.moba_decode_workspace_size.argtypes = [P]
        lib.moba_decode_workspace_size.restype = sz
        lib.moba_decode_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp]
        lib.moba_decode_fwd.restype = ctypes.c_int
        lib.moba_pool_last_block.argtypes = [P, vp, vp, vp]
        lib.moba_pool_last_block.restype = ctypes.c_int
        lib.moba_attn_naive.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        lib.moba_attn_naive.restype = ctypes.c_int
        lib.moba_gate_topk_noalloc.argtypes = [P, vp, vp, vp, vp]
        lib.moba_gate_topk_noalloc.restype = ctypes.c_int
        lib.moba_host_staging_size.argtypes = [P, ctypes.c_int]
        lib.moba_host_staging_size.restype = sz
        lib.moba_fwd_host.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        lib.moba_fwd_host.restype = ctypes.c_int
        lib.moba_launches_per_forward.argtypes = [P]
        lib.moba_launches_per_forward.restype = ctypes.c_int
        for f in ("moba_pool_keys", "moba_gate_topk", "moba_attn_fwd", "moba_fwd", "moba_route",
                  "moba_attn_past", "moba_attn_self_merge"):
            getattr(lib, f).restype = ctypes.c_int
        lib.moba_selftest_bounded_wait.argtypes = [ctypes.POINTER(ctypes.c_int32)]
        lib.moba_selftest_bounded_wait.restype = ctypes.c_int
        lib.moba_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int]
        lib.moba_read_device_error.restype = ctypes.c_int
        lib.moba_status_string.argtypes = [ctypes.c_int]
        lib.moba_status_string.restype = ctypes.c_char_p
        lib.moba_last_error.argtypes = []
        lib.moba_last_error.restype = ctypes.c_char_p
        _lib = lib
    return _lib


class MobaParams:
    """Host-side moba_params plus the buffers it points at (kept alive here)."""

    def __init__(self, cu_seqlens_host, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 block_size: int, top_k: int, cu_seqlens_device=None, softmax_scale: float = 0.0,
                 num_seqs: int | None = None, max_seqlen: int = 0):
        c = _CParams()
        if cu_seqlens_host is not None:
            self.cu_host = np.ascontiguousarray(np.asarray(cu_seqlens_host), dtype=np.int32)
            c.num_seqs = self.cu_host.size - 1
            c.cu_seqlens_host = self.cu_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
            if cu_seqlens_device is None:
                import torch
                cu_seqlens_device = torch.from_numpy(self.cu_host.copy()).cuda()
            self.cu_dev = cu_seqlens_device
            c.cu_seqlens = cu_seqlens_device.data_ptr()
            self.total_tokens = int(self.cu_host[-1])
        else:
            self.cu_host = None
            self.cu_dev = None
            c.num_seqs = int(num_seqs)
            c.max_seqlen = int(max_seqlen)
            self.total_tokens = int(num_seqs) * int(max_seqlen)
        c.num_q_heads = num_q_heads
        c.num_kv_heads = num_kv_heads
        c.head_dim = head_dim
        c.block_size = block_size
        c.top_k = top_k
        c.softmax_scale = softmax_scale
        self.c = c

    def ref(self):
        return ctypes.byref(self.c)

    @property
    def kbar_elems(self) -> int:
        return moba_kbar_elems(self)

    @property
    def workspace_bytes(self) -> int:
        return moba_workspace_size(self)

    @property
    def max_blocks(self) -> int:
        h, d = self.c.num_kv_heads, self.c.head_dim
        return self.kbar_elems // (self.c.num_seqs * h * d)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(rc: int):
    if rc != 0:
        raise MobaError(rc, load().moba_last_error().decode())


def moba_kbar_elems(p: MobaParams) -> int:
    return int(load().moba_kbar_elems(p.ref()))


def moba_workspace_size(p: MobaParams) -> int:
    return int(load().moba_workspace_size(p.ref()))


def moba_pool_keys(p: MobaParams, K, Kbar, stream=None) -> None:
    _check(load().moba_pool_keys(p.ref(), _ptr(K), _ptr(Kbar), _stream(stream)))


def moba_gate_topk(p: MobaParams, Q, Kbar, sel, workspace, stream=None) -> None:
    _check(load().moba_gate_topk(p.ref(), _ptr(Q), _ptr(Kbar), _ptr(sel), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def moba_attn_fwd(p: MobaParams, Q, K, V, sel, workspace, O, LSE, stream=None) -> None:
    _check(load().moba_attn_fwd(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(sel), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _ptr(O), _ptr(LSE),
                                _stream(stream)))


def moba_fwd(p: MobaParams, Q, K, V, workspace, O, LSE, Kbar=None, sel=None, stream=None) -> None:
    _check(load().moba_fwd(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kbar), _ptr(sel), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _ptr(O), _ptr(LSE),
                           _stream(stream)))


def moba_route(p: MobaParams, sel, workspace, stream=None) -> None:
    _check(load().moba_route(p.ref(), _ptr(sel), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))


def moba_attn_past(p: MobaParams, Q, K, V, workspace, stream=None) -> None:
    _check(load().moba_attn_past(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def moba_attn_self_merge(p: MobaParams, Q, K, V, sel, workspace, O, LSE, stream=None) -> None:
    _check(load().moba_attn_self_merge(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(sel), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(O), _ptr(LSE),
                                       _stream(stream)))


def moba_attn_naive(p: MobaParams, Q, K, V, sel, O, LSE, stream=None) -> None:
    """Mask-based attention over every causal key with the selection as a block mask
    (a baseline for moba_attn_fwd; same results up to rounding)."""
    _check(load().moba_attn_naive(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(sel), _ptr(O), _ptr(LSE),
                                  _stream(stream)))


def moba_bwd_workspace_size(p: MobaParams) -> int:
    return int(load().moba_bwd_workspace_size(p.ref()))


def moba_attn_bwd(p: MobaParams, Q, K, V, O, LSE, dO, sel, workspace, dQ, dK, dV, stream=None) -> None:
    """Gradients dQ [T,Hq,D], dK, dV [T,Hkv,D] (bf16) of MoBA attention for dO, with the
    forward's selection held fixed."""
    _check(load().moba_attn_bwd(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(dO), _ptr(sel),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dQ),
                                _ptr(dK), _ptr(dV), _stream(stream)))


def moba_decode_workspace_size(p: MobaParams) -> int:
    return int(load().moba_decode_workspace_size(p.ref()))


def moba_decode_fwd(p: MobaParams, Q, K, V, Kbar, workspace, O, LSE, sel=None, stream=None) -> None:
    """Gated decode: Q [num_seqs, Hq, D] (the newest token of each cached sequence) against
    the caches K, V [T, Hkv, D] described by p; O [num_seqs, Hq, D], LSE [num_seqs, Hq]."""
    _check(load().moba_decode_fwd(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kbar), _ptr(sel), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(O), _ptr(LSE),
                                  _stream(stream)))


def moba_pool_last_block(p: MobaParams, K, Kbar, stream=None) -> None:
    """Re-pool each sequence's last block into Kbar (after appending to a KV cache)."""
    _check(load().moba_pool_last_block(p.ref(), _ptr(K), _ptr(Kbar), _stream(stream)))


def moba_gate_topk_noalloc(p: MobaParams, Q, Kbar, sel, stream=None) -> None:
    """moba_gate_topk for callers without an allocator: scratch is a fixed array in the library."""
    _check(load().moba_gate_topk_noalloc(p.ref(), _ptr(Q), _ptr(Kbar), _ptr(sel), _stream(stream)))


def moba_host_staging_size(p: MobaParams, nstreams: int) -> int:
    return int(load().moba_host_staging_size(p.ref(), nstreams))


def moba_fwd_host(p: MobaParams, Q, K, V, O, LSE, staging, streams) -> None:
    """Forward on pinned HOST tensors (Q, K, V in; O, LSE out), copies overlapped with the
    kernels over the given CUDA streams; asynchronous (synchronise the streams afterwards)."""
    arr = (ctypes.c_void_p * len(streams))(*[_stream(s) for s in streams])
    _check(load().moba_fwd_host(p.ref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(staging),
                                staging.numel() * staging.element_size(), arr, len(streams)))


def moba_launches_per_forward(p: MobaParams) -> int:
    return int(load().moba_launches_per_forward(p.ref()))


def moba_read_device_error(clear: bool = False) -> int:
    """Device error word of the current device (non-zero: a kernel wait gave up)."""
    v = ctypes.c_int32(0)
    _check(load().moba_read_device_error(ctypes.byref(v), 1 if clear else 0))
    return int(v.value)


def moba_selftest_bounded_wait() -> int:
    """Run the bounded-wait failure path once; returns the device error word it produced."""
    v = ctypes.c_int32(0)
    _check(load().moba_selftest_bounded_wait(ctypes.byref(v)))
    return int(v.value)


def alloc_workspace(p: MobaParams, device="cuda"):
    import torch
    return torch.empty(max(p.workspace_bytes, 256), dtype=torch.uint8, device=device)


def moba_attention(Q, K, V, cu_seqlens_host, block_size: int, top_k: int, softmax_scale: float = 0.0,
                   workspace=None, stream=None):
    """MoBA causal prefill on packed bf16 Q [T,Hq,D], K/V [T,Hkv,D]; returns (O, LSE)."""
    import torch
    T, hq, D = Q.shape
    p = MobaParams(cu_seqlens_host, hq, K.shape[1], D, block_size, top_k, softmax_scale=softmax_scale)
    if workspace is None:
        workspace = alloc_workspace(p, Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty((T, hq), dtype=torch.float32, device=Q.device)
    moba_fwd(p, Q, K, V, workspace, O, LSE, stream=stream)
    return O, LSE
