"""ctypes front end for the fp64 C oracle (``gla_oracle.c``).

TEST INFRASTRUCTURE: used by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` only. Arrays are numpy float64, row-major:
q, k, log_a [B,H,L,K]; v, o, dO [B,H,L,V]; h0, hT, dhT, dh0 [B,H,K,V].

Layer definition (gla_oracle.c header): S_t = diag(exp(log_a_t)) S_{t-1} +
k_t^T v_t and o_t = q_t S_t -- the per-key-channel gate G_t = alpha_t^T 1 of
"Gated Linear Attention Transformers with Hardware-Efficient Training"
(atlas.scime.ai summary, section "Approach").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_SRC_GSA = os.path.join(_HERE, "gsa_oracle.c")
_LIB = os.path.join(_HERE, "libgla_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle (both C files) with gcc (OpenMP) into ``oracle/libgla_oracle.so``."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_GSA))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", _SRC, _SRC_GSA, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _declare(lib):
    lib.gla_oracle_fwd.argtypes = [_i64] * 5 + [_dp] * 7
    lib.gla_oracle_fwd.restype = None
    lib.gla_oracle_step.argtypes = [_i64] * 4 + [_dp] * 6
    lib.gla_oracle_step.restype = None
    lib.gla_oracle_bwd.argtypes = [_i64] * 5 + [_dp] * 13 + [_i64]
    lib.gla_oracle_bwd.restype = None
    lib.gsa_oracle_fwd.argtypes = [_i64] * 6 + [_dp] * 10
    lib.gsa_oracle_fwd.restype = None
    lib.gsa_oracle_bwd.argtypes = [_i64] * 6 + [_dp] * 15 + [_i64]
    lib.gsa_oracle_bwd.restype = None
    lib.gla_oracle_num_threads.restype = ctypes.c_int
    lib.gla_oracle_set_threads.argtypes = [ctypes.c_int]
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    with _lock:
        if _lib is None:
            build()
            _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def with_library(path: str):
    """The oracle's functions bound to another build of its C sources (the mutation tests load copies with
    a planted mistake to show that the pins catch it). Returns a namespace with fwd, bwd, step, gsa_fwd
    and gsa_bwd."""
    import functools
    import types

    lib = _declare(ctypes.CDLL(path))
    return types.SimpleNamespace(**{f.__name__: functools.partial(f, lib=lib)
                                    for f in (fwd, bwd, step, gsa_fwd, gsa_bwd)})


def _c(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.cast(None, _dp)
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    return int(_load().gla_oracle_num_threads())


def set_threads(n: int) -> None:
    _load().gla_oracle_set_threads(int(n))


def fwd(q, k, v, log_a, h0=None, lib=None):
    """Step recurrence forward. Returns (o [B,H,L,V], hT [B,H,K,V]) in fp64."""
    lib = _load(lib)
    q, k, v, log_a = _c(q), _c(k), _c(v), _c(log_a)
    B, H, L, K = q.shape
    V = v.shape[-1]
    assert k.shape == q.shape and log_a.shape == q.shape and v.shape == (B, H, L, V)
    h0c = None if h0 is None else _c(h0)
    if h0c is not None:
        assert h0c.shape == (B, H, K, V)
    o = np.zeros((B, H, L, V), np.float64)
    hT = np.zeros((B, H, K, V), np.float64)
    lib.gla_oracle_fwd(B, H, L, K, V, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(h0c), _ptr(o), _ptr(hT))
    return o, hT


def bwd(q, k, v, log_a, dO, h0=None, dhT=None, seg: int = 64, lib=None):
    """Reverse-mode gradients of <dO, o> + <dhT, hT>.

    Returns a dict with dq, dk, dv, dlog_a (direct chain rule), dlog_a_cf
    (closed form: reverse cumsum of q*dq - k*dk plus the dhT*hT term) and dh0.
    """
    lib = _load(lib)
    q, k, v, log_a, dO = _c(q), _c(k), _c(v), _c(log_a), _c(dO)
    B, H, L, K = q.shape
    V = v.shape[-1]
    h0c = None if h0 is None else _c(h0)
    dhTc = None if dhT is None else _c(dhT)
    dq = np.zeros((B, H, L, K))
    dk = np.zeros((B, H, L, K))
    dv = np.zeros((B, H, L, V))
    dla = np.zeros((B, H, L, K))
    dla_cf = np.zeros((B, H, L, K))
    dh0 = np.zeros((B, H, K, V))
    lib.gla_oracle_bwd(B, H, L, K, V, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(h0c), _ptr(dO), _ptr(dhTc),
                       _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dla_cf), _ptr(dh0), int(seg))
    return {"dq": dq, "dk": dk, "dv": dv, "dlog_a": dla, "dlog_a_cf": dla_cf, "dh0": dh0}


def step(q, k, v, log_a, S, lib=None):
    """One decode step. q,k,log_a [B,H,K]; v [B,H,V]; S [B,H,K,V].

    Returns (o [B,H,V], S_new); the input S is not modified.
    """
    lib = _load(lib)
    q, k, v, log_a = _c(q), _c(k), _c(v), _c(log_a)
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    B, H, K = q.shape
    V = v.shape[-1]
    o = np.zeros((B, H, V))
    lib.gla_oracle_step(B, H, K, V, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(S), _ptr(o))
    return o, S


# ---- gated slot attention (gsa_oracle.c) ------------------------------------------------------------
def gsa_fwd(q, k, v, log_a, hk0=None, hv0=None, lib=None):
    """Gated slot attention forward, step by step in fp64.

    q, k [B,H,L,K]; v [B,H,L,V]; log_a [B,H,L,m]; hk0 [B,H,m,K], hv0 [B,H,m,V] (None = zero).
    Returns (o [B,H,L,V], s [B,H,L,m] read weights, hkT [B,H,m,K], hvT [B,H,m,V]).
    """
    lib = _load(lib)
    q, k, v, log_a = _c(q), _c(k), _c(v), _c(log_a)
    B, H, L, K = q.shape
    V, m = v.shape[-1], log_a.shape[-1]
    assert k.shape == q.shape and v.shape == (B, H, L, V) and log_a.shape == (B, H, L, m)
    hk0c = None if hk0 is None else _c(hk0)
    hv0c = None if hv0 is None else _c(hv0)
    o = np.zeros((B, H, L, V))
    s = np.zeros((B, H, L, m))
    hkT = np.zeros((B, H, m, K))
    hvT = np.zeros((B, H, m, V))
    lib.gsa_oracle_fwd(B, H, L, K, V, m, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(hk0c), _ptr(hv0c), _ptr(o),
                       _ptr(s), _ptr(hkT), _ptr(hvT))
    return o, s, hkT, hvT


def gsa_bwd(q, k, v, log_a, dO, hk0=None, hv0=None, dhkT=None, dhvT=None, seg: int = 64, lib=None):
    """Reverse-mode gradients of <dO, o> + <dhkT, hkT> + <dhvT, hvT> for gated slot attention.

    Returns a dict with dq, dk, dv, dlog_a, dhk0, dhv0.
    """
    lib = _load(lib)
    q, k, v, log_a, dO = _c(q), _c(k), _c(v), _c(log_a), _c(dO)
    B, H, L, K = q.shape
    V, m = v.shape[-1], log_a.shape[-1]
    opt = [None if t is None else _c(t) for t in (hk0, hv0, dhkT, dhvT)]
    dq = np.zeros((B, H, L, K))
    dk = np.zeros((B, H, L, K))
    dv = np.zeros((B, H, L, V))
    dla = np.zeros((B, H, L, m))
    dhk0 = np.zeros((B, H, m, K))
    dhv0 = np.zeros((B, H, m, V))
    lib.gsa_oracle_bwd(B, H, L, K, V, m, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(opt[0]), _ptr(opt[1]),
                       _ptr(dO), _ptr(opt[2]), _ptr(opt[3]), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dhk0),
                       _ptr(dhv0), int(seg))
    return {"dq": dq, "dk": dk, "dv": dv, "dlog_a": dla, "dhk0": dhk0, "dhv0": dhv0}
