"""fp64 CPU oracle for the LightTransfer-Test prefill path (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` import this package.  The CUDA library never calls it and the
two share no code: this module is a thin ctypes wrapper over ``oracle.c`` (plain
C, fp64, libm), which it compiles with gcc on first use.

Every function takes bf16 tensors as numpy ``uint16`` bit patterns (shape
``[T, heads, d]``) and host ``int32`` ``cu_seqlens`` of length ``batch + 1``.
What each one computes, and the passage of the LightTransfer pages it follows,
is stated in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, IEEE)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp,
                               "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def _configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    lib.oracle_attn.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u16p,
                                ctypes.c_double, _i32p, _i32p, ctypes.c_int64, _f64p, _f64p, ctypes.c_int]
    lib.oracle_lazy_ratio_rows.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p,
                                           _u16p, ctypes.c_double, ctypes.c_int, ctypes.c_int, _i32p, _i32p,
                                           ctypes.c_int64, _f64p, ctypes.c_int, _f64p, ctypes.c_int]
    lib.oracle_lazy_ratio.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, _u16p,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _f64p,
                                      ctypes.c_int]
    lib.oracle_layer_scores.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p]
    lib.oracle_select_layers.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _u8p, _i32p]
    lib.oracle_queue_online.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _i32p, _i32p,
                                        ctypes.POINTER(ctypes.c_int)]
    lib.oracle_compact_kv.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u8p,
                                      ctypes.c_int, ctypes.c_int, _u16p, _u16p, _i32p]
    lib.oracle_attn_keys.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u16p, _i32p,
                                     ctypes.c_double, _f64p, _f64p]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def _check_bf16(x, name):
    if x.dtype != np.uint16 or x.ndim != 3 or not x.flags.c_contiguous:
        raise ValueError(f"{name} must be a C-contiguous uint16 [T, heads, d] array of bf16 bits")


def _cu(cu_seqlens):
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    if cu.ndim != 1 or cu.size < 2:
        raise ValueError("cu_seqlens must be int32 [batch+1]")
    return cu


def default_scale(d: int) -> float:
    """1/sqrt(d): the usual attention scale (the pages do not state another)."""
    return 1.0 / math.sqrt(d)


def all_items(cu_seqlens, hq):
    """(tokens, heads) covering every query row of every head."""
    T = int(cu_seqlens[-1])
    tokens = np.tile(np.arange(T, dtype=np.int32), hq)
    heads = np.repeat(np.arange(hq, dtype=np.int32), T)
    return tokens, heads


def attn(cu_seqlens, Q, K, V, scale=None, tokens=None, heads=None, nthreads=None):
    """Causal GQA attention rows.  Returns (O [n, d] float64, LSE [n] float64).

    Without ``tokens``/``heads`` every row is computed and the result is
    reshaped to O [T, hq, d] and LSE [hq, T].
    """
    for x, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _check_bf16(x, n)
    cu = _cu(cu_seqlens)
    T, hq, d = Q.shape
    hkv = K.shape[1]
    full = tokens is None
    if full:
        tokens, heads = all_items(cu, hq)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    n = tokens.size
    O = np.empty((n, d), np.float64)
    LSE = np.empty((n,), np.float64)
    rc = _load().oracle_attn(_ptr(cu, _i32p), cu.size - 1, hq, hkv, d, _ptr(Q, _u16p), _ptr(K, _u16p),
                             _ptr(V, _u16p), default_scale(d) if scale is None else float(scale),
                             _ptr(tokens, _i32p), _ptr(heads, _i32p), n, _ptr(O, _f64p), _ptr(LSE, _f64p),
                             _threads(nthreads))
    if rc:
        raise ValueError(f"oracle_attn failed ({rc})")
    if full:
        O = O.reshape(hq, T, d).transpose(1, 0, 2).copy()
        LSE = LSE.reshape(hq, T)
    return O, LSE


def lazy_ratio_rows(cu_seqlens, Q, K, S, W, tokens, heads, scale=None, lse=None, route="A", nthreads=None):
    """Per-row lazy ratio r_i for the listed (token, head) items (float64 [n])."""
    _check_bf16(Q, "Q")
    _check_bf16(K, "K")
    cu = _cu(cu_seqlens)
    T, hq, d = Q.shape
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    lse_a = None if lse is None else np.ascontiguousarray(lse, dtype=np.float64)
    if lse_a is not None and lse_a.size != tokens.size:
        raise ValueError("lse must hold one value per item")
    r = np.empty((tokens.size,), np.float64)
    rc = _load().oracle_lazy_ratio_rows(_ptr(cu, _i32p), cu.size - 1, hq, K.shape[1], d, _ptr(Q, _u16p),
                                        _ptr(K, _u16p), default_scale(d) if scale is None else float(scale),
                                        int(S), int(W), _ptr(tokens, _i32p), _ptr(heads, _i32p), tokens.size,
                                        _ptr(lse_a, _f64p), {"A": 0, "B": 1}[route], _ptr(r, _f64p),
                                        _threads(nthreads))
    if rc:
        raise ValueError(f"oracle_lazy_ratio_rows failed ({rc})")
    return r


def lazy_ratio(cu_seqlens, Q, K, S, W, n_obs, scale=None, lse=None, nthreads=None):
    """ratio [batch, hq] float64: mean of r_i over the last min(n_obs, N_b) rows.

    ``lse`` (optional) is an LSE array [hq, T]; when given it is used as the
    denominator instead of the oracle's own LSE.
    """
    _check_bf16(Q, "Q")
    _check_bf16(K, "K")
    cu = _cu(cu_seqlens)
    T, hq, d = Q.shape
    lse_a = None if lse is None else np.ascontiguousarray(lse, dtype=np.float64)
    if lse_a is not None and lse_a.shape != (hq, T):
        raise ValueError("lse must be [hq, T]")
    out = np.empty((cu.size - 1, hq), np.float64)
    rc = _load().oracle_lazy_ratio(_ptr(cu, _i32p), cu.size - 1, hq, K.shape[1], d, _ptr(Q, _u16p),
                                   _ptr(K, _u16p), default_scale(d) if scale is None else float(scale), int(S),
                                   int(W), int(n_obs), _ptr(lse_a, _f64p), _ptr(out, _f64p), _threads(nthreads))
    if rc:
        raise ValueError(f"oracle_lazy_ratio failed ({rc})")
    return out


def layer_scores(ratios):
    """ratios [L, batch, hq] -> scores [batch, L] (mean over query heads)."""
    r = np.ascontiguousarray(ratios, dtype=np.float64)
    L, B, H = r.shape
    out = np.empty((B, L), np.float64)
    if _load().oracle_layer_scores(_ptr(r, _f64p), L, B, H, _ptr(out, _f64p)):
        raise ValueError("oracle_layer_scores failed")
    return out


def select_layers(scores, budget):
    """Offline selection of one sequence: (lazy [L] uint8, order [budget] int32)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    L = s.size
    lazy = np.empty((L,), np.uint8)
    order = np.empty((max(budget, 1),), np.int32)
    if _load().oracle_select_layers(_ptr(s, _f64p), L, int(budget), _ptr(lazy, _u8p), _ptr(order, _i32p)):
        raise ValueError("oracle_select_layers failed")
    return lazy, order[:budget]


def queue_online(scores, budget, push_order=None):
    """Online queue of one sequence: the popped layers in pop order (int32)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    L = s.size
    po = None if push_order is None else np.ascontiguousarray(push_order, dtype=np.int32)
    popped = np.empty((max(L, 1),), np.int32)
    n = ctypes.c_int(0)
    if _load().oracle_queue_online(_ptr(s, _f64p), L, int(budget), _ptr(po, _i32p), _ptr(popped, _i32p),
                                   ctypes.byref(n)):
        raise ValueError("oracle_queue_online failed")
    return popped[: n.value].copy()


def compact_kv(cu_seqlens, K, V, mask, S, W, Ks=None, Vs=None):
    """Streaming KV of the masked sequences: (Ks, Vs [batch, hkv, S+W, d] uint16, len [batch] int32).

    ``Ks``/``Vs`` may be given pre-filled; rows of unmasked sequences are left as
    they are.
    """
    _check_bf16(K, "K")
    _check_bf16(V, "V")
    cu = _cu(cu_seqlens)
    B = cu.size - 1
    T, hkv, d = K.shape
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    if Ks is None:
        Ks = np.zeros((B, hkv, S + W, d), np.uint16)
    if Vs is None:
        Vs = np.zeros((B, hkv, S + W, d), np.uint16)
    ln = np.empty((B,), np.int32)
    if _load().oracle_compact_kv(_ptr(cu, _i32p), B, hkv, d, _ptr(K, _u16p), _ptr(V, _u16p), _ptr(m, _u8p),
                                 int(S), int(W), _ptr(Ks, _u16p), _ptr(Vs, _u16p), _ptr(ln, _i32p)):
        raise ValueError("oracle_compact_kv failed")
    return Ks, Vs, ln


def attn_keys(q, K, V, m, scale=None):
    """Attention of each query row over its own key rows (decode over a
    streaming cache).  q [n, d], K/V [n, m_max, d] uint16 bf16 bits, m [n] keys
    used per item.  Returns (O [n, d] float64, LSE [n] float64)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    m = np.ascontiguousarray(m, dtype=np.int32)
    n, d = q.shape
    if K.shape != V.shape or K.shape[0] != n or K.shape[2] != d or m.shape != (n,):
        raise ValueError("q [n, d], K/V [n, m_max, d], m [n]")
    O = np.empty((n, d), np.float64)
    LSE = np.empty((n,), np.float64)
    rc = _load().oracle_attn_keys(n, K.shape[1], d, _ptr(q, _u16p), _ptr(K, _u16p), _ptr(V, _u16p), _ptr(m, _i32p),
                                  default_scale(d) if scale is None else float(scale), _ptr(O, _f64p), _ptr(LSE, _f64p))
    if rc:
        raise ValueError(f"oracle_attn_keys failed ({rc})")
    return O, LSE
