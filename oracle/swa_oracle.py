"""ctypes wrapper around the C oracle (test infrastructure; see package docstring).

Inputs are numpy arrays holding either bf16 bit patterns (dtype uint16) or
float64 values; outputs are float64. Shapes: q/dO ``[B, T, H, D]``, k/v
``[B, T, Hk, D]`` with Hk dividing H (query head h reads K/V head h // (H // Hk);
Hk = H is plain multi-head attention), lse ``[B, H, T]``; decode q ``[B, H, D]``,
caches ``[B, cap, Hk, D]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "libswa_oracle.so")
_lock = threading.Lock()
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile swa_oracle.c into libswa_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_oracle())
            vp, L, d, dp, lp, ip = (ctypes.c_void_p, ctypes.c_long, ctypes.c_double,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p)
            lib.swa_oracle_fwd.argtypes = [vp, vp, vp, ctypes.c_int, L, L, L, L, L, L, d, dp, dp]
            lib.swa_oracle_fwd_rows.argtypes = [vp, vp, vp, ctypes.c_int, L, L, L, L, L, L, d, L, lp, dp, dp]
            lib.swa_oracle_bwd.argtypes = [vp, vp, vp, vp, ctypes.c_int, L, L, L, L, L, L, d, dp, dp, dp]
            lib.swa_oracle_dq_rows.argtypes = [vp, vp, vp, vp, ctypes.c_int, L, L, L, L, L, L, d, L, lp, dp]
            lib.swa_oracle_dkv_rows.argtypes = [vp, vp, vp, vp, ctypes.c_int, L, L, L, L, L, L, d, L, lp, dp, dp]
            lib.swa_oracle_decode.argtypes = [vp, vp, vp, ctypes.c_int, ip, L, L, L, L, L, L, d, dp, dp]
            for f in ("swa_oracle_fwd", "swa_oracle_fwd_rows", "swa_oracle_bwd", "swa_oracle_dq_rows",
                      "swa_oracle_dkv_rows", "swa_oracle_decode"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def oracle_threads() -> int:
    """Number of OpenMP threads the oracle will use (OMP_NUM_THREADS, else all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.strip().isdigit():
        return int(env)
    return os.cpu_count() or 1


def _prep(*arrays):
    """Validate dtype agreement; return (contiguous arrays, in_bf16 flag)."""
    dt = arrays[0].dtype
    if dt not in (np.uint16, np.float64):
        raise TypeError("oracle inputs must be bf16 bits (uint16) or float64")
    out = []
    for a in arrays:
        if a.dtype != dt:
            raise TypeError("all oracle inputs must share one dtype")
        out.append(np.ascontiguousarray(a))
    return out, int(dt == np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _kv_heads(H: int, kv) -> int:
    """K/V head count of a K or V array (axis 2), which must divide the query head count H."""
    Hk = kv.shape[2]
    if Hk < 1 or H % Hk != 0:
        raise ValueError(f"K/V heads ({Hk}) must divide query heads ({H})")
    return Hk


def oracle_fwd(q, k, v, W: int, scale: float | None = None):
    """Full forward. Returns (o [B,T,H,D] f64, lse [B,H,T] f64)."""
    (q, k, v), bf = _prep(q, k, v)
    B, T, H, D = q.shape
    Hk = _kv_heads(H, k)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    o = np.empty((B, T, H, D), np.float64)
    lse = np.empty((B, H, T), np.float64)
    _load().swa_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), bf, B, T, H, Hk, D, int(W), float(scale), _ptr(o), _ptr(lse))
    return o, lse


def oracle_fwd_rows(q, k, v, W: int, rows, scale: float | None = None):
    """Forward on selected rows; rows = int array [n, 3] of (b, h, i). Returns (o [n,D], lse [n])."""
    (q, k, v), bf = _prep(q, k, v)
    B, T, H, D = q.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    idx = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = idx.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    _load().swa_oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), bf, B, T, H, _kv_heads(H, k), D, int(W), float(scale),
                                n, _ptr(idx), _ptr(o), _ptr(lse))
    return o, lse


def oracle_bwd(q, k, v, do, W: int, scale: float | None = None):
    """Full backward. Returns (dq [B,T,H,D], dk [B,T,Hk,D], dv [B,T,Hk,D]) f64."""
    (q, k, v, do), bf = _prep(q, k, v, do)
    B, T, H, D = q.shape
    Hk = _kv_heads(H, k)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    dq = np.empty((B, T, H, D), np.float64)
    dk = np.empty((B, T, Hk, D), np.float64)
    dv = np.empty_like(dk)
    _load().swa_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), bf, B, T, H, Hk, D, int(W), float(scale),
                           _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def oracle_dq_rows(q, k, v, do, W: int, rows, scale: float | None = None):
    """dQ on selected query rows (b, h, i). Returns [n, D] f64."""
    (q, k, v, do), bf = _prep(q, k, v, do)
    B, T, H, D = q.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    idx = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    dq = np.empty((idx.shape[0], D), np.float64)
    _load().swa_oracle_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), bf, B, T, H, _kv_heads(H, k), D, int(W),
                               float(scale),
                               idx.shape[0], _ptr(idx), _ptr(dq))
    return dq


def oracle_dkv_rows(q, k, v, do, W: int, rows, scale: float | None = None):
    """dK, dV on selected key rows (b, hk, j), hk a K/V head. Returns (dk [n,D], dv [n,D]) f64."""
    (q, k, v, do), bf = _prep(q, k, v, do)
    B, T, H, D = q.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    idx = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    dk = np.empty((idx.shape[0], D), np.float64)
    dv = np.empty_like(dk)
    _load().swa_oracle_dkv_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), bf, B, T, H, _kv_heads(H, k), D, int(W),
                                float(scale),
                                idx.shape[0], _ptr(idx), _ptr(dk), _ptr(dv))
    return dk, dv


def oracle_decode(q, k_cache, v_cache, cache_len, W: int, scale: float | None = None):
    """Decode. q [B,H,D], caches [B,cap,Hk,D], cache_len [B] int. Returns (o [B,H,D], lse [B,H]) f64."""
    (q, k_cache, v_cache), bf = _prep(q, k_cache, v_cache)
    B, H, D = q.shape
    cap = k_cache.shape[1]
    Hk = _kv_heads(H, k_cache)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    cl = np.ascontiguousarray(np.asarray(cache_len, dtype=np.int32))
    if cl.shape != (B,) or cl.min(initial=1) < 1 or cl.max(initial=1) > cap:
        raise ValueError("cache_len must be [B] with values in [1, cap]")
    o = np.empty((B, H, D), np.float64)
    lse = np.empty((B, H), np.float64)
    _load().swa_oracle_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), bf, cl.ctypes.data_as(ctypes.c_void_p),
                              B, cap, H, Hk, D, int(W), float(scale), _ptr(o), _ptr(lse))
    return o, lse


def oracle_prefill(q, k_new, v_new, k_cache, v_cache, cache_len, W: int, scale: float | None = None):
    """Chunked prefill with append, written out as its definition (the engine's
    flash_attn_with_kvcache with new K / V, apidog guide section 6): for sequence b the cache
    afterwards holds its first cache_len[b] tokens followed by the chunk, and the chunk's query t
    is row cache_len[b] + t of the forward over that token sequence.

    q [B,Tn,H,D]; k_new, v_new [B,Tn,Hk,D]; caches [B,cap,Hk,D]; cache_len [B] (tokens cached
    before the chunk).  Returns (o [B,Tn,H,D], lse [B,H,Tn], k_cache_after, v_cache_after); the
    inputs are not modified and cache slots past cache_len[b] + Tn keep their input values."""
    (q, k_new, v_new, k_cache, v_cache), _ = _prep(q, k_new, v_new, k_cache, v_cache)
    B, Tn, H, D = q.shape
    cap = k_cache.shape[1]
    kc, vc = k_cache.copy(), v_cache.copy()
    o = np.empty((B, Tn, H, D), np.float64)
    lse = np.empty((B, H, Tn), np.float64)
    for b in range(B):
        L = int(cache_len[b])
        n = L + Tn
        if L < 0 or n > cap:
            raise ValueError("cache_len[b] + Tn must lie in [Tn, cap]")
        kc[b, L:n] = k_new[b]
        vc[b, L:n] = v_new[b]
        qs = np.zeros((1, n, H, D), dtype=q.dtype)
        qs[0, L:] = q[b]
        rows = np.array([(0, h, L + t) for h in range(H) for t in range(Tn)], dtype=np.int64)
        ob, lb = oracle_fwd_rows(qs, kc[b:b + 1, :n], vc[b:b + 1, :n], W, rows, scale)
        o[b] = ob.reshape(H, Tn, D).transpose(1, 0, 2)
        lse[b] = lb.reshape(H, Tn)
    return o, lse, kc, vc
