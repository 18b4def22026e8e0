"""fp64 CPU oracle for exact softmax attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  It wraps ``ra_oracle.cpp`` (plain C++ built with gcc) through ctypes and
shares nothing with the CUDA library.

Functions
---------
attention(q, k, v, causal, rows=None, threads=1)
    The plain definition softmax(Q K^T / sqrt(D)) V in fp64 (causal mask on original positions,
    diagonal included), on all rows or on a per-(b, h) row subset.  Returns (out, lse) as float64
    numpy arrays: out [B, H, n_rows, D] and lse [B, H, n_rows].
ring_blockwise(q, k, v, n_ring, causal, layout)
    The ring loop of the ultralytics.com toy (query block i fixed, key/value block
    j = (i - s) mod N at step s), with max subtraction and token layouts, in fp64.
    Returns (out [B, S, H, D], lse [B, H, S], block_pairs [N, N]).
merge(m, l, O, m2, l2, O2)
    Online-softmax merge identities (troisinh.com "Ring Attention", "Tai sao no hoat dong").
layout_positions(S, n_ring, layout)
    Global position of each (shard, local index) under a layout, shape [N, S/N].
attention_varlen(q, k, v, cu_seqlens, causal, threads=1)
    The plain definition for sequences packed along the token axis of q, k, v [1, S_total, H, D]
    (sequence k = tokens cu[k]..cu[k+1]-1).  Returns out [S_total, H, D] and lse [H, S_total].
rope(x, pos_offset=0, base=10000.0)
    Rotary embedding with global positions (troisinh.com "Ring Attention", "RoPE va Position
    Embedding"), pairs (2p, 2p+1) rotated by m * base^(-2p/D), in fp64.  Returns [B, S, H, D].
attention_backward(q, k, v, dout, causal, threads=1)
    Gradients (dq, dk, dv) of the plain definition for the upstream gradient dout, in fp64, each
    [B, S, H, D] (troisinh.com "Ring Attention", "Blockwise Backward"; chain rule written out).
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ra_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libra_oracle.so")

LAYOUTS = {"contiguous": 0, "striped": 1, "zigzag": 2}
_DTYPE_CODES = {np.dtype(np.float32): 0, np.dtype(np.uint16): 1, np.dtype(np.float64): 2}


def build(src=_SRC, out=_LIB_PATH):
    """Compile the oracle with gcc (plain -O2, no fast-math: fp64 as written)."""
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def load(path=None):
    """Load (building first if needed) the oracle shared library."""
    path = path or _LIB_PATH
    if path == _LIB_PATH and (not os.path.exists(path)
                              or os.path.getmtime(path) < os.path.getmtime(_SRC)):
        build()
    lib = ctypes.CDLL(path)
    i64, vp, dp = ctypes.c_int64, ctypes.c_void_p, ctypes.POINTER(ctypes.c_double)
    lib.ora_attention.restype = ctypes.c_int
    lib.ora_attention.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, ctypes.c_int,
                                  vp, i64, vp, vp, ctypes.c_int]
    lib.ora_ring_blockwise.restype = ctypes.c_int
    lib.ora_ring_blockwise.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64,
                                       ctypes.c_int, ctypes.c_int, vp, vp, vp]
    lib.ora_merge.restype = None
    lib.ora_merge.argtypes = [i64, i64, dp, dp, dp, dp, dp, dp]
    lib.ora_layout_positions.restype = ctypes.c_int
    lib.ora_layout_positions.argtypes = [i64, i64, ctypes.c_int, vp]
    lib.ora_attention_varlen.restype = ctypes.c_int
    lib.ora_attention_varlen.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, ctypes.c_int, vp, i64, vp, vp,
                                         ctypes.c_int]
    lib.ora_rope.restype = ctypes.c_int
    lib.ora_rope.argtypes = [vp, ctypes.c_int, i64, i64, i64, i64, i64, ctypes.c_double, vp]
    lib.ora_attention_backward.restype = ctypes.c_int
    lib.ora_attention_backward.argtypes = [vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i64,
                                           ctypes.c_int, vp, vp, vp, ctypes.c_int]
    return lib


_lib = None


def _get():
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def _as_input(x):
    """Host array for the oracle: float32, float64, or bf16 passed as its raw uint16 bits.

    Accepts numpy arrays or CPU torch tensors (bf16 tensors are reinterpreted, not converted).
    """
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16)
            return np.ascontiguousarray(x.numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x)


def _code(arr):
    if arr.dtype not in _DTYPE_CODES:
        raise TypeError(f"oracle input dtype {arr.dtype} not supported")
    return _DTYPE_CODES[arr.dtype]


def attention(q, k, v, causal, rows=None, threads=1, lib=None):
    lib = lib or _get()
    q, k, v = _as_input(q), _as_input(k), _as_input(v)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    B, S, H, D = q.shape
    if rows is None:
        n_rows = S
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        if rows_arr.ndim == 1:
            rows_arr = np.ascontiguousarray(np.broadcast_to(rows_arr, (B * H, rows_arr.size)))
        rows_arr = rows_arr.reshape(B * H, -1)
        n_rows = rows_arr.shape[1]
    out = np.empty((B, H, n_rows, D), dtype=np.float64)
    lse = np.empty((B, H, n_rows), dtype=np.float64)
    rc = lib.ora_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, _code(q), B, H, S, D,
                           int(bool(causal)),
                           None if rows_arr is None else rows_arr.ctypes.data, n_rows,
                           out.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("ora_attention rejected its arguments")
    return out, lse


def ring_blockwise(q, k, v, n_ring, causal, layout="contiguous", lib=None):
    lib = lib or _get()
    q, k, v = _as_input(q), _as_input(k), _as_input(v)
    B, S, H, D = q.shape
    out = np.empty((B, S, H, D), dtype=np.float64)
    lse = np.empty((B, H, S), dtype=np.float64)
    pairs = np.zeros((n_ring, n_ring), dtype=np.int64)
    rc = lib.ora_ring_blockwise(q.ctypes.data, k.ctypes.data, v.ctypes.data, _code(q), B, H, S,
                                D, n_ring, int(bool(causal)), LAYOUTS[layout], out.ctypes.data,
                                lse.ctypes.data, pairs.ctypes.data)
    if rc != 0:
        raise ValueError("ora_ring_blockwise rejected its arguments")
    return out, lse, pairs


def merge(m, l, O, m2, l2, O2, lib=None):
    """Merge (m2, l2, O2) into copies of (m, l, O); O is the un-normalised accumulator [n, D]."""
    lib = lib or _get()
    m = np.array(m, dtype=np.float64).ravel()
    l = np.array(l, dtype=np.float64).ravel()
    O = np.array(O, dtype=np.float64).reshape(m.size, -1).copy()
    m2 = np.ascontiguousarray(np.asarray(m2, dtype=np.float64).ravel())
    l2 = np.ascontiguousarray(np.asarray(l2, dtype=np.float64).ravel())
    O2 = np.ascontiguousarray(np.asarray(O2, dtype=np.float64).reshape(m.size, -1))
    dp = ctypes.POINTER(ctypes.c_double)
    ptr = lambda a: a.ctypes.data_as(dp)
    lib.ora_merge(m.size, O.shape[1], ptr(m), ptr(l), ptr(O), ptr(m2), ptr(l2), ptr(O2))
    return m, l, O


def layout_positions(S, n_ring, layout, lib=None):
    lib = lib or _get()
    pos = np.empty((n_ring, S // n_ring), dtype=np.int64)
    if lib.ora_layout_positions(S, n_ring, LAYOUTS[layout], pos.ctypes.data) != 0:
        raise ValueError("layout does not split S evenly")
    return pos


def attention_backward(q, k, v, dout, causal, threads=1, lib=None):
    """fp64 gradients (dq, dk, dv), each [B, S, H, D], of softmax(Q K^T / sqrt(D)) V for dout."""
    lib = lib or _get()
    q, k, v, dout = _as_input(q), _as_input(k), _as_input(v), _as_input(dout)
    if not (q.dtype == k.dtype == v.dtype == dout.dtype):
        raise TypeError("q, k, v, dout must share a dtype")
    B, S, H, D = q.shape
    dq, dk, dv = (np.empty((B, S, H, D), dtype=np.float64) for _ in range(3))
    rc = lib.ora_attention_backward(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data,
                                    _code(q), B, H, S, D, int(bool(causal)), dq.ctypes.data,
                                    dk.ctypes.data, dv.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("ora_attention_backward rejected its arguments")
    return dq, dk, dv


def rope(x, pos_offset=0, base=10000.0, lib=None):
    """fp64 rotary embedding of x [B, S, H, D]; token g takes the position g + pos_offset."""
    lib = lib or _get()
    x = _as_input(x)
    B, S, H, D = x.shape
    y = np.empty((B, S, H, D), dtype=np.float64)
    if lib.ora_rope(x.ctypes.data, _code(x), B, S, H, D, int(pos_offset), float(base), y.ctypes.data) != 0:
        raise ValueError("ora_rope rejected its arguments")
    return y


def attention_varlen(q, k, v, cu_seqlens, causal, threads=1, lib=None):
    """fp64 attention of packed sequences: q, k, v [1, S_total, H, D]; returns (out [S_total, H, D],
    lse [H, S_total])."""
    lib = lib or _get()
    q, k, v = _as_input(q), _as_input(k), _as_input(v)
    if q.shape[0] != 1:
        raise ValueError("packed sequences take batch 1")
    _, S, H, D = q.shape
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    out = np.empty((S, H, D), dtype=np.float64)
    lse = np.empty((H, S), dtype=np.float64)
    rc = lib.ora_attention_varlen(q.ctypes.data, k.ctypes.data, v.ctypes.data, _code(q), S, H, D,
                                  int(bool(causal)), cu.ctypes.data, cu.size - 1, out.ctypes.data,
                                  lse.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("ora_attention_varlen rejected its arguments")
    return out, lse
