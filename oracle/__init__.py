"""fp64 CPU oracle for block-sparse paged GQA attention (forward, and the
gradients of its output).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library: the arithmetic lives in ``gbsa_oracle.c`` (plain loops,
fp64, a two-pass softmax over exactly the selected, unmasked keys), compiled
here with gcc; ``scheduler.py`` is an independent sequential rebuild of the
work-list format the metadata kernel writes.

What the oracle computes is stated at the top of ``gbsa_oracle.c``; it follows
the GenericBlockSparseAttention article (cf-1.com/news/4865651), "Function /
sparse attention mechanism" and "Constraints", and the FlashAttention blog
post on CANN ops-transformer (ai6s.net), "three steps" (the online softmax is
exactly the two-pass softmax).  Pins: tests/test_oracle_pins.py (forward),
tests/test_oracle_backward.py (gradients: finite differences, closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gbsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libgbsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compiles gbsa_oracle.c into _build/libgbsa_oracle.so (gcc, -O2)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        compile_to(_SRC, _LIB_PATH)
    return _LIB_PATH


def compile_to(src: str, dst: str) -> str:
    """Compiles an oracle C source file into a shared library at ``dst``."""
    tmp = dst + f".{os.getpid()}.tmp"
    # -ffp-contract=off keeps every product and sum a separately rounded fp64 op.
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-pthread", src, "-o", tmp, "-lm"])
    os.replace(tmp, dst)
    return dst


def load_library(path: str):
    """Loads an oracle shared library and declares its entry point."""
    lib = ctypes.CDLL(path)
    f = lib.gbsa_oracle_attention_rows
    i32, i64, dbl, ptr = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    f.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, i64, dbl, i32, i32, i32,
                  ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, i64, ptr, ptr, ptr, ptr, i32]
    f.restype = ctypes.c_int
    w = lib.gbsa_oracle_widen
    w.argtypes = [i32, ptr, i64, ptr]
    w.restype = ctypes.c_int
    g = lib.gbsa_oracle_attention_backward
    g.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, i64, dbl, i32, i32, i32,
                  ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                  ptr]
    g.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _as(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


DTYPES = {"bf16": 0, "fp16": 1}


def widen(bits, dtype="bf16", lib=None):
    """Exact float64 values of 16-bit patterns of ``dtype`` ("bf16" / "fp16")."""
    b = _as(bits, np.uint16).reshape(-1)
    out = np.empty(b.size, np.float64)
    if (lib or _load()).gbsa_oracle_widen(DTYPES[dtype], _ptr(b), b.size, _ptr(out)) != 0:
        raise ValueError(dtype)
    return out.reshape(np.shape(bits))


def attention_rows(*, q_bits, k_bits, v_bits, kv_page_stride, num_pages, sparse_idx, sparse_count,
                   cu_seqlens_q, seqused_q, seqused_kv, block_table, block_x, scale,
                   win_left=-1, win_right=-1, rows, dtype="bf16", cu_seqlens_kv=None,
                   out_abs=None, gap_abs=None, n_threads=None, lib=None):
    """Reference out/lse for selected (token, head) rows.

    q_bits:  uint16 [T, N1, D] -- bit patterns of the queries, bf16 or fp16
             (``dtype``); k_bits and v_bits use the same type.
    k_bits, v_bits: flat uint16 arrays of the page pool; page ``p`` row ``r``
             head ``h`` starts at ``p*kv_page_stride + (r*N2 + h)*D``.  With
             ``cu_seqlens_kv`` they are TND instead: position ``p`` of
             sequence ``b``, head ``h`` starts at ``((cu_seqlens_kv[b]+p)*N2 + h)*D``
             (block_table, num_pages, kv_page_stride unused).
    rows:    int64 [n, 2] -- (global token index, query head).
    out_abs: optional float64 [n, D] array filled with sum_p w_p |v_p[d]|.
    gap_abs: optional float64 [n, D] array filled with sum_p w_p (m - s_p) |v_p[d]|
             (m the row's largest score s_p, natural-log units).
    Returns (out [n, D] float64, lse [n] float64).  Rows past seqused_q, or
    with no visible key, give out = 0 and lse = -inf.
    """
    q_bits = _as(q_bits, np.uint16)
    k_bits = _as(k_bits, np.uint16).reshape(-1)
    v_bits = _as(v_bits, np.uint16).reshape(-1)
    T, N1, D = q_bits.shape
    sparse_idx = _as(sparse_idx, np.int32)
    N2, tqb, top_k = sparse_idx.shape
    sparse_count = _as(sparse_count, np.int32)
    cu = _as(cu_seqlens_q, np.int64)
    squ = _as(seqused_q, np.int32)
    sku = _as(seqused_kv, np.int32)
    cukv = _as(cu_seqlens_kv, np.int64)
    B = cu.shape[0] - 1
    if cukv is None:
        bt = _as(block_table, np.int32)
        max_pages = bt.shape[1]
        need = (num_pages - 1) * kv_page_stride + 128 * N2 * D
    else:
        bt, max_pages, num_pages, kv_page_stride = None, 0, 0, 0
        need = int(cukv[-1]) * N2 * D
    if k_bits.size < need or v_bits.size < need:
        raise ValueError("page pool arrays are shorter than num_pages pages")
    rows = _as(rows, np.int64).reshape(-1, 2)
    n = rows.shape[0]
    out = np.zeros((n, D), np.float64)
    lse = np.full((n,), -np.inf, np.float64)
    for name, a in (("out_abs", out_abs), ("gap_abs", gap_abs)):
        if a is not None and (a.shape != (n, D) or a.dtype != np.float64
                              or not a.flags.c_contiguous):
            raise ValueError(f"{name}: expected a contiguous float64 [n, D] array")
    rc = (lib or _load()).gbsa_oracle_attention_rows(
        B, T, N1, N2, D, block_x, tqb, top_k, max_pages, num_pages, kv_page_stride, float(scale),
        win_left, win_right, DTYPES[dtype], _ptr(q_bits), _ptr(k_bits), _ptr(v_bits), _ptr(sparse_idx),
        _ptr(sparse_count), _ptr(cu), _ptr(squ), _ptr(sku), _ptr(bt), _ptr(cukv), _ptr(rows), n,
        _ptr(out), _ptr(lse), None if out_abs is None else _ptr(out_abs),
        None if gap_abs is None else _ptr(gap_abs), n_threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle rejected the inputs (code {rc})")
    return out, lse


def attention(*, q_bits, rows=None, **kw):
    """Reference out [T, N1, D] and lse [T, N1] (fp64) over every row."""
    T, N1, D = np.asarray(q_bits).shape
    tt, hh = np.meshgrid(np.arange(T), np.arange(N1), indexing="ij")
    all_rows = np.stack([tt.reshape(-1), hh.reshape(-1)], axis=1)
    out, lse = attention_rows(q_bits=q_bits, rows=all_rows, **kw)
    return out.reshape(T, N1, D), lse.reshape(T, N1)


def attention_backward(*, q_bits, k_bits, v_bits, dout_bits, kv_page_stride, num_pages, sparse_idx,
                       sparse_count, cu_seqlens_q, seqused_q, seqused_kv, block_table, block_x,
                       scale, win_left=-1, win_right=-1, dtype="bf16", cu_seqlens_kv=None,
                       with_abs=False, lib=None):
    """Reference gradients of out (fp64) for an incoming gradient ``dout_bits``
    (uint16 [T, N1, D], the type of q).  Arguments as for ``attention_rows``.

    Returns (dq [T, N1, D], dk, dv), dk and dv flat float64 arrays laid out
    like k_bits and v_bits (the page pool with ``kv_page_stride``, or TND);
    with ``with_abs`` also (dq_abs, dk_abs, dv_abs), the same sums of the
    absolute values of their terms.
    """
    q_bits = _as(q_bits, np.uint16)
    dout_bits = _as(dout_bits, np.uint16)
    k_bits = _as(k_bits, np.uint16).reshape(-1)
    v_bits = _as(v_bits, np.uint16).reshape(-1)
    T, N1, D = q_bits.shape
    if dout_bits.shape != q_bits.shape:
        raise ValueError("dout: expected the shape of q")
    sparse_idx = _as(sparse_idx, np.int32)
    N2, tqb, top_k = sparse_idx.shape
    sparse_count = _as(sparse_count, np.int32)
    cu = _as(cu_seqlens_q, np.int64)
    squ = _as(seqused_q, np.int32)
    sku = _as(seqused_kv, np.int32)
    cukv = _as(cu_seqlens_kv, np.int64)
    B = cu.shape[0] - 1
    if cukv is None:
        bt = _as(block_table, np.int32)
        max_pages = bt.shape[1]
        need = (num_pages - 1) * kv_page_stride + 128 * N2 * D
    else:
        bt, max_pages, num_pages, kv_page_stride = None, 0, 0, 0
        need = int(cukv[-1]) * N2 * D
    if k_bits.size < need or v_bits.size < need:
        raise ValueError("page pool arrays are shorter than num_pages pages")
    dq = np.zeros((T, N1, D), np.float64)
    dk = np.zeros(k_bits.size, np.float64)
    dv = np.zeros(v_bits.size, np.float64)
    absv = [np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)] if with_abs else [None] * 3
    rc = (lib or _load()).gbsa_oracle_attention_backward(
        B, T, N1, N2, D, block_x, tqb, top_k, max_pages, num_pages, kv_page_stride, float(scale),
        win_left, win_right, DTYPES[dtype], _ptr(q_bits), _ptr(k_bits), _ptr(v_bits),
        _ptr(dout_bits), _ptr(sparse_idx), _ptr(sparse_count), _ptr(cu), _ptr(squ), _ptr(sku),
        _ptr(bt), _ptr(cukv), _ptr(dq), _ptr(dk), _ptr(dv), *(_ptr(a) for a in absv))
    if rc != 0:
        raise ValueError(f"oracle rejected the inputs (code {rc})")
    return (dq, dk, dv, *absv) if with_abs else (dq, dk, dv)

