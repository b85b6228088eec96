"""CPU oracle of the HGRN2 recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and
reference legs) may import this package.  The product library never does, and
the two share no code: the oracle is ``oracle.c`` (plain sequential fp64 loops,
see its header for the equations and their source) plus ``brute.py`` (an
independent quadratic-form restatement in NumPy for tiny inputs).

This module only marshals NumPy arrays to ``oracle.c`` through ctypes and
builds ``liboracle.so`` with gcc when it is missing or stale.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2 -fopenmp); returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ci = ctypes.c_int
        lib.oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, ci, ci, ci, ci, ci]
        lib.oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, ci, ci, ci, ci, ci]
        lib.oracle_step.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci]
        lib.oracle_sd_fwd.argtypes = [dp] * 7 + [ci] * 5
        lib.oracle_sd_bwd.argtypes = [dp] * 12 + [ci] * 5
        lib.oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def fwd(q, log_f, i, h0=None):
    """o [B,T,H,dv] and hT [B,H,dk,dv] of the recurrence, in fp64.

    q, log_f: [B,T,H,dk]; i: [B,T,H,dv]; h0: [B,H,dk,dv] or None (zeros)."""
    q, log_f, i, h0 = _f64(q), _f64(log_f), _f64(i), _f64(h0)
    B, T, H, dk = q.shape
    dv = i.shape[-1]
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    _load().oracle_fwd(_p(q), _p(log_f), _p(i), _p(h0), _p(o), _p(hT), B, T, H, dk, dv)
    return o, hT


def bwd(q, log_f, i, dO, h0=None, dhT=None, want_dk=False):
    """Gradients (dq, dlog_f, di, dh0[, dk]) of L = <o, dO> + <hT, dhT>, in fp64."""
    q, log_f, i, dO, h0, dhT = (_f64(a) for a in (q, log_f, i, dO, h0, dhT))
    B, T, H, dk = q.shape
    dv = i.shape[-1]
    dq = np.zeros_like(q)
    dlf = np.zeros_like(q)
    di = np.zeros_like(i)
    dh0 = np.zeros((B, H, dk, dv))
    dkk = np.zeros_like(q) if want_dk else None
    _load().oracle_bwd(_p(q), _p(log_f), _p(i), _p(h0), _p(dO), _p(dhT),
                       _p(dq), _p(dlf), _p(di), _p(dh0), _p(dkk), B, T, H, dk, dv)
    if want_dk:
        return dq, dlf, di, dh0, dkk
    return dq, dlf, di, dh0


def step(q, log_f, i, S):
    """One decode step.  q, log_f: [B,H,dk]; i: [B,H,dv]; S: [B,H,dk,dv].

    Returns (o [B,H,dv], S_new); the input S is not modified."""
    q, log_f, i = _f64(q), _f64(log_f), _f64(i)
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    B, H, dk = q.shape
    dv = i.shape[-1]
    o = np.zeros((B, H, dv))
    _load().oracle_step(_p(q), _p(log_f), _p(i), _p(S), _p(o), B, H, dk, dv)
    return o, S


def lower_bound_log_f(g, lb: float):
    """log f for the lower-bounded forget gate f = lb + (1 - lb) * sigmoid(g), in fp64.

    ("HGRN2: Gated Linear RNNs with State Expansion", §2.2: the forget gate of each layer is
    kept above a learnable lower bound lb in [0, 1).)  Written as
        log f = log(1 + lb e^{-g}) - log(1 + e^{-g}),
    both terms through log-add-exp, so that neither g -> +inf nor g -> -inf overflows; lb = 0
    gives log sigmoid(g)."""
    g = np.asarray(g, dtype=np.float64)
    if lb == 0.0:
        return -np.logaddexp(0.0, -g)
    return np.logaddexp(0.0, np.log(lb) - g) - np.logaddexp(0.0, -g)


def step_bwd(q, log_f, i, S, dO, dS=None):
    """Gradients (dq, dlog_f, di, dS_prev) of one decode step, for L = <o, dO> + <S_new, dS>
    with (o, S_new) = step(q, log_f, i, S).  One step is the recurrence over a single token
    starting from h0 = S, so this is bwd() at T = 1 with h0 = S and dhT = dS.

    q, log_f: [B,H,dk]; i, dO: [B,H,dv]; S, dS: [B,H,dk,dv] (dS None: zero)."""
    dq, dlf, di, dS0 = bwd(_f64(q)[:, None], _f64(log_f)[:, None], _f64(i)[:, None], _f64(dO)[:, None],
                           h0=S, dhT=dS)
    return dq[:, 0], dlf[:, 0], di[:, 0], dS0


def lower_bound_dlog_f_dg(g, lb: float):
    """d log f / d g of the lower-bounded gate (see lower_bound_log_f), in fp64.

    f = lb + (1 - lb) sigmoid(g) gives df/dg = (1 - lb) sigmoid(g) sigmoid(-g), and
    d log f / dg = (df/dg) / f.  With u = e^{-|g|} in (0, 1] this is
        (1 - lb) u / ((1 + u) (1 + lb u))     for g >= 0,
        (1 - lb) u / ((1 + u) (lb + u))       for g < 0,
    a ratio of positive terms, so it keeps full relative precision in both tails."""
    g = np.asarray(g, dtype=np.float64)
    u = np.exp(-np.abs(g))
    den = np.where(g >= 0, (1.0 + u) * (1.0 + lb * u), (1.0 + u) * (lb + u))
    return (1.0 - lb) * u / den


def sd_fwd(q, k, v, log_g, h0=None):
    """Scalar-decay variant, in fp64: S_t = g_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t with
    g_t = exp(log_g_t) one decay per (batch, token, head) (the per-head decay of Mamba2/RetNet
    that "HGRN2: Gated Linear RNNs with State Expansion", §5, contrasts with its per-dimension
    decay).  q, k: [B,T,H,dk]; v: [B,T,H,dv]; log_g: [B,T,H]; h0: [B,H,dk,dv] or None.
    Returns (o [B,T,H,dv], hT)."""
    q, k, v, log_g, h0 = (_f64(a) for a in (q, k, v, log_g, h0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    _load().oracle_sd_fwd(_p(q), _p(k), _p(v), _p(log_g), _p(h0), _p(o), _p(hT), B, T, H, dk, dv)
    return o, hT


def sd_bwd(q, k, v, log_g, dO, h0=None, dhT=None):
    """Gradients (dq, dk, dv, dlog_g, dh0) of L = <o, dO> + <hT, dhT> for sd_fwd, in fp64
    (back-propagation through time)."""
    q, k, v, log_g, dO, h0, dhT = (_f64(a) for a in (q, k, v, log_g, dO, h0, dhT))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dq, dk_, dv_ = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg = np.zeros_like(log_g)
    dh0 = np.zeros((B, H, dk, dv))
    _load().oracle_sd_bwd(_p(q), _p(k), _p(v), _p(log_g), _p(h0), _p(dO), _p(dhT), _p(dq), _p(dk_), _p(dv_),
                          _p(dg), _p(dh0), B, T, H, dk, dv)
    return dq, dk_, dv_, dg, dh0
