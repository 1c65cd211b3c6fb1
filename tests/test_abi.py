"""The C-ABI library loads, exports every entry point its header declares, and rejects
bad arguments on the host before touching CUDA (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_gate_b200 as mb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "moba.h")).read()
    return re.findall(r"MOBA_API\s+[\w\s\*]*?\b(moba_\w+)\s*\(", txt)


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("moba_pool_keys", "moba_gate_topk", "moba_attn_fwd", "moba_fwd", "moba_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = mb.load()
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) >= set(mb.EXPORTS)


def test_sizes_are_host_computations():
    p = mb.MobaParams(None, 32, 8, 128, 2048, 3, num_seqs=1, max_seqlen=1 << 20)
    assert p.kbar_elems == 512 * 8 * 128
    ws = p.workspace_bytes
    R = (1 << 20) * 32 * 2
    assert ws >= R * 128 * 2 + R * 8 + (1 << 20) * 32 * 3 * 4  # fp16 partial rows, LSE, row ids, sel
    # varlen: MB follows the longest sequence
    q = mb.MobaParams.__new__(mb.MobaParams)
    cu = np.array([0, 131072, 196608, 229376, 245760], dtype=np.int32)
    c = mb._CParams()
    c.num_seqs = 4
    c.cu_seqlens_host = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    c.cu_seqlens = 256  # device pointer is not dereferenced by the size queries
    c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.top_k = 32, 8, 128, 512, 12
    q.c = c
    assert mb.moba_kbar_elems(q) == 4 * 256 * 8 * 128


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, 2), ("block_size", 100, 2), ("block_size", 16384, 2), ("top_k", 0, 2),
    ("top_k", 17, 2), ("num_kv_heads", 3, 1), ("num_seqs", 0, 1)])
def test_bad_params_are_rejected_before_any_cuda_call(field, value, status):
    p = mb.MobaParams(None, 4, 2, 128, 128, 3, num_seqs=1, max_seqlen=256)
    setattr(p.c, field, value)
    assert mb.moba_workspace_size(p) == 0
    lib = mb.load()
    rc = lib.moba_pool_keys(p.ref(), 16, 16, None)
    assert rc == status
    assert lib.moba_last_error()


def test_bad_cu_seqlens_rejected():
    lib = mb.load()
    for cu in ([1, 5], [0, 5, 3]):
        arr = np.array(cu, dtype=np.int32)
        c = mb._CParams()
        c.num_seqs = len(cu) - 1
        c.cu_seqlens_host = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        c.cu_seqlens = 256
        c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.top_k = 2, 1, 64, 128, 3
        assert lib.moba_pool_keys(ctypes.byref(c), 16, 16, None) == 1


def test_misaligned_pointers_rejected():
    p = mb.MobaParams(None, 2, 1, 64, 128, 3, num_seqs=1, max_seqlen=256)
    lib = mb.load()
    assert lib.moba_pool_keys(p.ref(), 18, 16, None) == 3
    assert lib.moba_pool_keys(p.ref(), None, 16, None) == 1
    ws = p.workspace_bytes
    assert lib.moba_gate_topk(p.ref(), 16, 16, 16, 256, ws - 1, None) == 4
    assert lib.moba_gate_topk(p.ref(), 16, 16, 16, 272, ws, None) == 4


def test_empty_problem_is_a_no_op():
    p = mb.MobaParams(None, 2, 1, 64, 128, 3, num_seqs=1, max_seqlen=0)
    lib = mb.load()
    assert lib.moba_fwd(p.ref(), None, None, None, None, None, None, 0, None, None, None) == 0


def test_host_staging_is_per_slot_group_sized():
    # one slot holds one KV-head group's Q, K, V, O, LSE and that group's workspace
    p = mb.MobaParams(None, 32, 8, 128, 2048, 3, num_seqs=1, max_seqlen=1 << 16)
    one = mb.moba_host_staging_size(p, 1)
    assert one > 0 and mb.moba_host_staging_size(p, 3) == 3 * one
    T, G, D = 1 << 16, 4, 128
    group_io = T * G * D * 2 * 2 + T * D * 2 * 2 + T * G * 4  # Q and O, K and V, LSE
    g = mb.MobaParams(None, G, 1, D, 2048, 3, num_seqs=1, max_seqlen=T)
    assert group_io + g.workspace_bytes <= one <= group_io + g.workspace_bytes + 8 * 256
    assert mb.moba_host_staging_size(p, 0) == 0


def test_backward_and_decode_workspace_sizes():
    # backward: routing arrays as in the forward, Dp (T*Hq fp32), one fp32 dQ partial per routed slot
    T, hq, hkv, D, bs, k = 1 << 16, 32, 8, 128, 2048, 3
    p = mb.MobaParams(None, hq, hkv, D, bs, k, num_seqs=1, max_seqlen=T)
    R = T * hq * (k - 1)
    bw = mb.moba_bwd_workspace_size(p)
    assert R * D * 4 + T * hq * 4 + R * 4 <= bw <= R * D * 4 + T * hq * 4 + R * 4 + (R // 256 + 64) * 4 * 260 + 8 * 256
    # decode: an fp32 partial O, its LSE and a selection slot per (sequence, head, slot)
    q = mb.MobaParams(None, hq, hkv, D, bs, k, num_seqs=64, max_seqlen=T)
    units = 64 * hq * k
    assert mb.moba_decode_workspace_size(q) == (units * D * 4 + 255) // 256 * 256 + 2 * ((units * 4 + 255) // 256 * 256)


def test_decode_rejects_empty_caches_before_any_cuda_call():
    lib = mb.load()
    arr = np.array([0, 5, 5, 9], dtype=np.int32)  # the second sequence is empty
    c = mb._CParams()
    c.num_seqs = 3
    c.cu_seqlens_host = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    c.cu_seqlens = 256
    c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.top_k = 2, 1, 64, 128, 3
    rc = lib.moba_decode_fwd(ctypes.byref(c), 16, 16, 16, 16, None, 256, 1 << 20, 16, 16, None)
    assert rc == 1 and b"empty" in lib.moba_last_error()
    p = mb.MobaParams(None, 2, 1, 64, 128, 3, num_seqs=2, max_seqlen=0)
    assert lib.moba_decode_fwd(p.ref(), 16, 16, 16, 16, None, 256, 1 << 20, 16, 16, None) == 1


def test_backward_and_naive_check_arguments_before_any_cuda_call():
    lib = mb.load()
    p = mb.MobaParams(None, 2, 1, 64, 128, 3, num_seqs=1, max_seqlen=256)
    ws = mb.moba_bwd_workspace_size(p)
    # a NULL gradient, a misaligned output, a short workspace
    assert lib.moba_attn_bwd(p.ref(), 16, 16, 16, 16, 16, None, 16, 256, ws, 16, 16, 16, None) == 1
    assert lib.moba_attn_bwd(p.ref(), 16, 16, 16, 16, 16, 16, 16, 256, ws, 16, 18, 16, None) == 3
    assert lib.moba_attn_bwd(p.ref(), 16, 16, 16, 16, 16, 16, 16, 256, ws - 1, 16, 16, 16, None) == 4
    assert lib.moba_attn_naive(p.ref(), 16, 16, 16, None, 16, 16, None) == 1
    assert lib.moba_pool_last_block(p.ref(), 18, 16, None) == 3
