"""Python wrapper of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module; the product path (the
CUDA library and its binding) never does.  It shares no code with the CUDA
path: it builds and loads its own C file and takes plain numpy arrays.

Inputs are numpy arrays of bf16 *bit patterns* (``np.uint16``) so that the
oracle sees exactly the values the GPU sees; the C side widens them to
double without rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` with gcc into ``oracle/_build/liboracle.so``."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _declare(lib):
    P = ctypes.c_void_p
    i = ctypes.c_int
    lib.oracle_paged_attention.argtypes = [i, i, i, i, i, i, i, P, P, P, P, P, P,
                                           ctypes.c_double, P, P, i]
    lib.oracle_paged_attention.restype = i
    lib.oracle_paged_attention_rows.argtypes = [i, i, i, i, i, i, i, P, P, P, P, P, P,
                                                ctypes.c_double, P, P, ctypes.c_long, P, P, i]
    lib.oracle_paged_attention_rows.restype = i
    lib.oracle_paged_attention_mode.argtypes = [i, i, i, i, i, i, i, P, P, P, P, P, P,
                                                ctypes.c_double, i, P, P, i]
    lib.oracle_paged_attention_mode.restype = i
    lib.oracle_paged_attention_fp8.argtypes = [i, i, i, i, i, i, i, P, P, P, ctypes.c_double,
                                               ctypes.c_double, P, P, P, ctypes.c_double, P, P, i]
    lib.oracle_paged_attention_fp8.restype = i
    lib.oracle_e4m3_decode.argtypes = [P, ctypes.c_long, P]
    lib.oracle_e4m3_decode.restype = None
    lib.oracle_merge_states.argtypes = [i, i, P, P, P, P]
    lib.oracle_merge_states.restype = None
    lib.oracle_append_kv.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P]
    lib.oracle_append_kv.restype = i
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def load_library(path: str):
    """Load another build of ``oracle.c`` (the tests build copies with a
    planted mistake to show that the pins catch it)."""
    return _declare(ctypes.CDLL(path))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns, got %s" % a.dtype)
    return a


def _i32(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.int32)


def default_threads() -> int:
    return os.cpu_count() or 1


def paged_attention(q, k_pool, v_pool, page_table, seq_lens, cu_q_lens, scale,
                    num_pages: int = 0, nthreads: int | None = None, lib=None,
                    causal: bool = True):
    """All rows.  Shapes: q [T, Hq, D]; pools [P, ps, Hkv, D]; page_table [B, C];
    seq_lens [B]; cu_q_lens [B+1] or None (one query token per request).
    ``causal=False`` lets every row see all of its request's keys.
    Returns (out [T, Hq, D] float64, lse [T, Hq] float64)."""
    q, k_pool, v_pool = _u16(q), _u16(k_pool), _u16(v_pool)
    page_table, seq_lens, cu_q_lens = _i32(page_table), _i32(seq_lens), _i32(cu_q_lens)
    T, Hq, D = q.shape
    _, ps, Hkv, D2 = k_pool.shape
    assert D2 == D and v_pool.shape == k_pool.shape
    B, C = page_table.shape
    out = np.zeros((T, Hq, D), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    L = lib or _load()
    if causal:
        rc = L.oracle_paged_attention(
            B, Hq, Hkv, D, ps, C, int(num_pages), _ptr(q), _ptr(k_pool), _ptr(v_pool),
            _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), float(scale), _ptr(out),
            _ptr(lse), int(nthreads or default_threads()))
    else:
        rc = L.oracle_paged_attention_mode(
            B, Hq, Hkv, D, ps, C, int(num_pages), _ptr(q), _ptr(k_pool), _ptr(v_pool),
            _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), float(scale), 0, _ptr(out),
            _ptr(lse), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: %s" % {1: "live page id out of range",
                                         2: "out of memory"}.get(rc, rc))
    return out, lse


def paged_attention_rows(q, k_pool, v_pool, page_table, seq_lens, cu_q_lens, scale,
                         row_t, row_h, num_pages: int = 0, nthreads: int | None = None,
                         lib=None):
    """Only the rows (row_t[u], row_h[u]).  Returns (out [n, D], lse [n])."""
    q, k_pool, v_pool = _u16(q), _u16(k_pool), _u16(v_pool)
    page_table, seq_lens, cu_q_lens = _i32(page_table), _i32(seq_lens), _i32(cu_q_lens)
    row_t, row_h = _i32(row_t), _i32(row_h)
    T, Hq, D = q.shape
    _, ps, Hkv, _ = k_pool.shape
    B, C = page_table.shape
    n = int(row_t.shape[0])
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = (lib or _load()).oracle_paged_attention_rows(
        B, Hq, Hkv, D, ps, C, int(num_pages), _ptr(q), _ptr(k_pool), _ptr(v_pool),
        _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), float(scale), _ptr(row_t),
        _ptr(row_h), n, _ptr(out), _ptr(lse), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: %s" % {1: "live page id out of range",
                                         2: "out of memory"}.get(rc, rc))
    return out, lse


def merge_states(o_s, lse_s):
    """Merge partial states of one row: o_s [n, D] (each normalised over its
    own keys), lse_s [n].  Returns (o [D], lse)."""
    o_s = np.ascontiguousarray(o_s, dtype=np.float64)
    lse_s = np.ascontiguousarray(lse_s, dtype=np.float64)
    n, D = o_s.shape
    o = np.zeros((D,), dtype=np.float64)
    lse = np.zeros((1,), dtype=np.float64)
    _load().oracle_merge_states(n, D, _ptr(o_s), _ptr(lse_s), _ptr(o), _ptr(lse))
    return o, float(lse[0])


def append_kv(k_new, v_new, k_pool, v_pool, page_table, seq_lens, cu_q_lens, num_pages=0):
    """Paged KV append (see ``oracle_append_kv``).  k_new / v_new: bf16 bits
    [T, Hkv, D]; the pools ([P, ps, Hkv, D] bf16 bits) are copied and the
    copies returned with the new rows written, plus the flag mask."""
    k_new = _u16(k_new)
    v_new = _u16(v_new)
    k_out = _u16(k_pool).copy()
    v_out = _u16(v_pool).copy()
    page_table = _i32(page_table)
    seq_lens = _i32(seq_lens)
    cu = None if cu_q_lens is None else _i32(cu_q_lens)
    P_, ps, Hkv, D = k_out.shape
    B, C = page_table.shape
    flags = _load().oracle_append_kv(B, Hkv, D, ps, C, int(num_pages), _ptr(k_new), _ptr(v_new),
                                     _ptr(k_out), _ptr(v_out), _ptr(page_table), _ptr(seq_lens),
                                     _ptr(cu))
    return k_out, v_out, int(flags)


def e4m3_decode(codes):
    """E4M3 codes (uint8) -> float64 values, as the oracle reads fp8 pools."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(codes.shape, dtype=np.float64)
    _load().oracle_e4m3_decode(_ptr(codes), codes.size, _ptr(out))
    return out


def paged_attention_fp8(q, k8, v8, k_scale, v_scale, page_table, seq_lens, cu_q_lens, scale,
                        num_pages: int = 0, nthreads: int | None = None, lib=None):
    """Causal attention over E4M3 pools (uint8 codes [P, ps, Hkv, D]) with
    per-tensor descales; q as bf16 bits.  Returns (out, lse) in float64."""
    q = _u16(q)
    k8 = np.ascontiguousarray(k8, dtype=np.uint8)
    v8 = np.ascontiguousarray(v8, dtype=np.uint8)
    page_table, seq_lens, cu_q_lens = _i32(page_table), _i32(seq_lens), _i32(cu_q_lens)
    T, Hq, D = q.shape
    _, ps, Hkv, D2 = k8.shape
    assert D2 == D and v8.shape == k8.shape
    B, C = page_table.shape
    out = np.zeros((T, Hq, D), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    rc = (lib or _load()).oracle_paged_attention_fp8(
        B, Hq, Hkv, D, ps, C, int(num_pages), _ptr(q), _ptr(k8), _ptr(v8), float(k_scale),
        float(v_scale), _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), float(scale),
        _ptr(out), _ptr(lse), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: %s" % {1: "live page id out of range",
                                         2: "out of memory"}.get(rc, rc))
    return out, lse
