"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library never links or calls it, and it shares
no code with the CUDA library.  The arithmetic lives in ``attn_oracle.c`` (plain C,
fp64, OpenMP over (sequence, head)); this module only builds it and marshals numpy
arrays.

Layout conventions (the same as the C file): q/k/v/o are packed token-major
``[T, H, d]`` arrays; a dense ``[B, N, H, d]`` batch is passed as ``T = B*N`` with
``cu = [0, N, 2N, ...]``.  LSE comes back as ``[H, T]``.

Pins (what fixes this oracle to something other than itself) live in
``tests/test_oracle_pins.py``.  ``oracle_online_fwd``'s conditional-rescale rule is
a reading of the pages (see the C file); every function here is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        ip = ctypes.POINTER(ctypes.c_int)
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.oracle_fwd.argtypes = [dp, dp, dp, dp, dp, ci, i64p, ci, ci, ci, cd, ci]
        lib.oracle_fwd.restype = ci
        lib.oracle_fwd_rows.argtypes = [dp, dp, dp, ci, i64p, ci, ci, ci, cd, i64p, ip, ci,
                                        dp, dp, ci]
        lib.oracle_fwd_rows.restype = ci
        lib.oracle_probs.argtypes = [dp, dp, ci, i64p, ci, ci, ci, cd, ci, ci, dp]
        lib.oracle_probs.restype = ci
        lib.oracle_fwd_masked.argtypes = [dp, dp, dp, dp, dp, ci, i64p, ci, ci, ci, ci, ci, cd, ci]
        lib.oracle_fwd_masked.restype = ci
        lib.oracle_fwd_rows_masked.argtypes = [dp, dp, dp, ci, i64p, ci, ci, ci, ci, ci, cd, i64p,
                                               ip, ci, dp, dp, ci]
        lib.oracle_fwd_rows_masked.restype = ci
        lib.oracle_probs_masked.argtypes = [dp, dp, ci, i64p, ci, ci, ci, ci, ci, cd, ci, ci, dp]
        lib.oracle_probs_masked.restype = ci
        lib.oracle_online_fwd.argtypes = [dp, dp, dp, dp, dp, ci, i64p, ci, ci, ci, cd, ci, ci, cd]
        lib.oracle_online_fwd.restype = ctypes.c_int64
        lib.oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, ci, i64p, ci, ci, ci, cd, ci]
        lib.oracle_bwd.restype = ci
        lib.oracle_bwd_masked.argtypes = [dp, dp, dp, dp, dp, dp, dp, ci, i64p, ci, ci, ci, ci, ci,
                                          cd, ci]
        lib.oracle_bwd_masked.restype = ci
        lib.oracle_bwd_sampled.argtypes = [dp, dp, dp, dp, ci, i64p, ci, ci, ci, cd, ci, ci,
                                           ip, ci, ip, ci, dp, dp, dp, ci]
        lib.oracle_bwd_sampled.restype = ci
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Contiguous fp64 copy of a numpy array or CPU torch tensor (exact for bf16)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _cu(cu, T: int) -> np.ndarray:
    cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int64))
    if cu.ndim != 1 or cu.size < 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu must be a non-decreasing prefix-sum array from 0 to T")
    return cu


def dense_cu(B: int, N: int) -> np.ndarray:
    return np.arange(B + 1, dtype=np.int64) * N


def _window(window):
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    return wl, wr


def fwd(q, k, v, cu, causal: bool, scale: float, nthreads: int = 0, window=None):
    """Exact forward: returns (o [T,H,d] fp64, lse [H,T] fp64, threads used).

    ``window = (wl, wr)`` adds the sliding-window mask: key j is visible to query i
    only if ``i - wl <= j <= i + wr`` (a negative bound is unbounded)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, d = q.shape
    cu = _cu(cu, T)
    o = np.zeros_like(q)
    lse = np.zeros((H, T), dtype=np.float64)
    wl, wr = _window(window)
    used = _load().oracle_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), cu.size - 1,
                                     _ptr(cu, ctypes.c_int64), H, d, int(causal), wl, wr,
                                     float(scale), int(nthreads))
    if used < 0:
        raise ValueError("oracle_fwd rejected its arguments")
    return o, lse, used


def fwd_rows(q, k, v, cu, causal: bool, scale: float, rows, heads, nthreads: int = 0,
             window=None):
    """Exact forward for selected (token, head) rows: returns (o [R,d], lse [R])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, d = q.shape
    cu = _cu(cu, T)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    heads = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    if rows.shape != heads.shape or rows.ndim != 1:
        raise ValueError("rows and heads must be 1-D of equal length")
    o = np.zeros((rows.size, d), dtype=np.float64)
    lse = np.zeros(rows.size, dtype=np.float64)
    wl, wr = _window(window)
    rc = _load().oracle_fwd_rows_masked(_ptr(q), _ptr(k), _ptr(v), cu.size - 1,
                                        _ptr(cu, ctypes.c_int64), H, d, int(causal), wl, wr,
                                        float(scale), _ptr(rows, ctypes.c_int64),
                                        _ptr(heads, ctypes.c_int), rows.size, _ptr(o), _ptr(lse),
                                        int(nthreads))
    if rc < 0:
        raise ValueError("oracle_fwd_rows rejected its arguments")
    return o, lse


def probs(q, k, cu, causal: bool, scale: float, b: int, h: int, window=None) -> np.ndarray:
    """Probability matrix P [L, L] of sequence b, head h."""
    q, k = _f64(q), _f64(k)
    T, H, d = q.shape
    cu = _cu(cu, T)
    L = int(cu[b + 1] - cu[b])
    P = np.zeros((L, L), dtype=np.float64)
    wl, wr = _window(window)
    rc = _load().oracle_probs_masked(_ptr(q), _ptr(k), cu.size - 1, _ptr(cu, ctypes.c_int64), H,
                                     d, int(causal), wl, wr, float(scale), int(b), int(h), _ptr(P))
    if rc < 0:
        raise ValueError("oracle_probs rejected its arguments")
    return P


def online_fwd(q, k, v, cu, causal: bool, scale: float, Br: int, Bc: int, tau: float):
    """Tiled online softmax with conditional rescale (tau in natural-log units).
    Returns (o, lse, number of rescales)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, d = q.shape
    cu = _cu(cu, T)
    o = np.zeros_like(q)
    lse = np.zeros((H, T), dtype=np.float64)
    n = _load().oracle_online_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), cu.size - 1,
                                  _ptr(cu, ctypes.c_int64), H, d, int(causal), float(scale),
                                  int(Br), int(Bc), float(tau))
    if n < 0:
        raise ValueError("oracle_online_fwd rejected its arguments")
    return o, lse, int(n)


def bwd(q, k, v, dout, cu, causal: bool, scale: float, nthreads: int = 0, window=None):
    """Textbook backward: returns (dq, dk, dv), each [T,H,d] fp64 (``window`` as
    for ``fwd``)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, H, d = q.shape
    cu = _cu(cu, T)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    wl, wr = _window(window)
    rc = _load().oracle_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                   _ptr(dv), cu.size - 1, _ptr(cu, ctypes.c_int64), H, d,
                                   int(causal), wl, wr, float(scale), int(nthreads))
    if rc < 0:
        raise ValueError("oracle_bwd rejected its arguments")
    return dq, dk, dv


def bwd_sampled(q, k, v, dout, cu, causal: bool, scale: float, b: int, h: int, q_rows, k_rows,
                nthreads: int = 0):
    """Backward at selected local query rows (dQ) and key rows (dK, dV) of sequence b,
    head h: returns (dq [nq,d], dk [nk,d], dv [nk,d]) in fp64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, H, d = q.shape
    cu = _cu(cu, T)
    qi = np.ascontiguousarray(np.asarray(q_rows, dtype=np.int32))
    kj = np.ascontiguousarray(np.asarray(k_rows, dtype=np.int32))
    dq = np.zeros((qi.size, d)); dk = np.zeros((kj.size, d)); dv = np.zeros((kj.size, d))
    rc = _load().oracle_bwd_sampled(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), cu.size - 1,
                                    _ptr(cu, ctypes.c_int64), H, d, int(causal), float(scale),
                                    int(b), int(h), _ptr(qi, ctypes.c_int), qi.size,
                                    _ptr(kj, ctypes.c_int), kj.size, _ptr(dq), _ptr(dk), _ptr(dv),
                                    int(nthreads))
    if rc < 0:
        raise ValueError("oracle_bwd_sampled rejected its arguments")
    return dq, dk, dv


def lse_to_dense(lse_ht: np.ndarray, B: int, N: int) -> np.ndarray:
    """[H, B*N] -> [B, H, N] (the dense LSE layout of the CUDA library)."""
    H = lse_ht.shape[0]
    return np.ascontiguousarray(lse_ht.reshape(H, B, N).transpose(1, 0, 2))
