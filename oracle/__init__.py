"""fp64 CPU oracle for exact softmax attention -- TEST INFRASTRUCTURE ONLY.

The CUDA library under ``exact_attention_110_b200`` is checked against this oracle. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it;
the product path never does, and this package imports nothing from the product.

The arithmetic lives in ``attn_ref.cpp`` (plain C++ fp64, OpenMP over rows). This module
only builds it and marshals numpy arrays.

Parity pins (see ``tests/test_oracle.py``): every function here is pinned against closed
forms, invariants, SciPy/Torch fp64 library routines and central finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attn_ref.cpp"
_LIB = _HERE / "liboracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile attn_ref.cpp into liboracle.so (g++ -O2 -fopenmp)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17", str(_SRC), "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB))
        dp = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_fwd.argtypes = [dp, dp, dp, i64, i32, i32, f64, i32, u8p, i32, dp, dp]
        lib.oracle_fwd_rows.argtypes = [dp, dp, dp, i32, i32, f64, i32, u8p, i32,
                                        ctypes.POINTER(ctypes.c_int), i32, dp, dp]
        lib.oracle_bwd.argtypes = [dp, dp, dp, dp, i64, i32, i32, f64, i32, u8p, i32, dp, dp, dp, dp]
        lib.oracle_online_fwd.argtypes = [dp, dp, dp, i64, i32, i32, f64, i32, u8p, i32, i32, i32, dp, dp]
        lib.oracle_fwd_qk.argtypes = [dp, dp, dp, i64, i32, i32, i32, f64, i32, dp, dp]
        lib.oracle_bwd_qk.argtypes = [dp, dp, dp, dp, i64, i32, i32, i32, f64, i32, dp, dp, dp, dp]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _mask_arg(mask, N: int, mask_bs: int):
    if mask is None:
        return None, None
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    nb = (N + mask_bs - 1) // mask_bs
    if m.shape != (nb, nb):
        raise ValueError(f"block mask must be {nb}x{nb}, got {m.shape}")
    return m, ctypes.c_void_p(m.ctypes.data)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _shape(q):
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = q.shape
    return B, H, N, d


def attention_fwd(q, k, v, scale: float, causal: bool = False, mask=None, mask_bs: int = 128):
    """Three-pass softmax attention. q, k, v: [B, H, N, d]. Returns (O [B,H,N,d], LSE [B,H,N])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape(q)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    m, mp = _mask_arg(mask, N, mask_bs)
    _load().oracle_fwd(_ptr(q), _ptr(k), _ptr(v), B * H, N, d, float(scale), int(causal), mp,
                       mask_bs, _ptr(o), _ptr(lse))
    return o, lse


def attention_fwd_qk(q, k, v, scale: float, causal: bool = False):
    """General shapes: q [B, H, Nq, d] against k, v [B, H, Nk, d] (bottom-right causal
    alignment: key j visible to query i iff j <= i + Nk - Nq). Returns (O, LSE)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = _shape(q)
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H and d")
    o = np.empty_like(q)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    _load().oracle_fwd_qk(_ptr(q), _ptr(k), _ptr(v), B * H, Nq, Nk, d, float(scale), int(causal), _ptr(o), _ptr(lse))
    return o, lse


def attention_fwd_rows(qh, kh, vh, rows, scale: float, causal: bool = False, mask=None, mask_bs: int = 128):
    """Forward for selected query rows of one head. qh, kh, vh: [N, d]."""
    qh, kh, vh = _f64(qh), _f64(kh), _f64(vh)
    N, d = qh.shape
    r = np.ascontiguousarray(rows, dtype=np.int32)
    o = np.empty((r.size, d), dtype=np.float64)
    lse = np.empty(r.size, dtype=np.float64)
    m, mp = _mask_arg(mask, N, mask_bs)
    _load().oracle_fwd_rows(_ptr(qh), _ptr(kh), _ptr(vh), N, d, float(scale), int(causal), mp, mask_bs,
                            r.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), r.size, _ptr(o), _ptr(lse))
    return o, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool = False, mask=None, mask_bs: int = 128):
    """Analytic backward. Returns (dQ, dK, dV, D) with D_i = sum_j P_ij dP_ij."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = _shape(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    D = np.empty((B, H, N), dtype=np.float64)
    m, mp = _mask_arg(mask, N, mask_bs)
    _load().oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B * H, N, d, float(scale), int(causal), mp,
                       mask_bs, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(D))
    return dq, dk, dv, D


def attention_bwd_qk(q, k, v, do, scale: float, causal: bool = False):
    """Analytic backward for general shapes (the gradient of attention_fwd_qk): q, do
    [B, H, Nq, d]; k, v [B, H, Nk, d]; bottom-right causal alignment. Returns (dQ, dK, dV, D)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, Nq, d = _shape(q)
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != k.shape or do.shape != q.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H and d; do must have q's shape")
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    D = np.empty((B, H, Nq), dtype=np.float64)
    _load().oracle_bwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B * H, Nq, Nk, d, float(scale), int(causal),
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(D))
    return dq, dk, dv, D


def attention_online_fwd(q, k, v, scale: float, block: int, deferred: bool, causal: bool = False,
                         mask=None, mask_bs: int = 128):
    """Block-by-block online-softmax forward (per-step normalised or deferred)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape(q)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    m, mp = _mask_arg(mask, N, mask_bs)
    _load().oracle_online_fwd(_ptr(q), _ptr(k), _ptr(v), B * H, N, d, float(scale), int(causal), mp,
                              mask_bs, int(block), int(deferred), _ptr(o), _ptr(lse))
    return o, lse
