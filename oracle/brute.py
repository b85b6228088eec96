"""Independent quadratic-form restatement of the HGRN2 recurrence (tiny inputs only).

TEST INFRASTRUCTURE ONLY (used by tests/ to pin the C oracle; never by the
product path).  It does not share code with ``oracle.c``: instead of stepping
the state, it writes every output as an explicit sum over past tokens, which is
the linear-attention reading of the recurrence ("HGRN2: Gated Linear RNNs with
State Expansion", §3.2: the recurrence equals gated linear attention with
key = 1 - forget gate, value = input, query = output gate; §5: one decay per key
dimension).

Unrolling S_t = Diag(f_t) S_{t-1} + k_t i_t^T from S_{-1} = h0, with
c_t = sum_{r<=t} log f_r (cumulative, per key dimension j):

    S_t[j,:] = exp(c_t[j]) h0[j,:] + sum_{s<=t} k_s[j] exp(c_t[j] - c_s[j]) i_s
    o_t      = sum_j q_t[j] S_t[j,:]

Because the decay is per key dimension, it stays inside the sum over j; only
when f is shared by all j does the textbook masked form ((Q K^T) * D) V with
D_ts = prod_{s<r<=t} f_r hold, and ``masked_attention_shared_decay`` writes
that form out literally for that case.
"""
from __future__ import annotations

import numpy as np


def quadratic_form(q, log_f, i, h0=None):
    """o and hT of one or more heads via the explicit double sum (float64)."""
    q = np.asarray(q, np.float64)
    a = np.asarray(log_f, np.float64)
    x = np.asarray(i, np.float64)
    B, T, H, dk = q.shape
    dv = x.shape[-1]
    k = -np.expm1(a)
    c = np.cumsum(a, axis=1)  # [B,T,H,dk], inclusive
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                acc = np.zeros(dv)
                if h0 is not None:
                    acc += (q[b, t, h] * np.exp(c[b, t, h])) @ np.asarray(h0, np.float64)[b, h]
                for s in range(t + 1):
                    w = np.sum(q[b, t, h] * k[b, s, h] * np.exp(c[b, t, h] - c[b, s, h]))
                    acc += w * x[b, s, h]
                o[b, t, h] = acc
            # final state, same unrolling at t = T-1
            S = np.zeros((dk, dv))
            if h0 is not None:
                S += np.exp(c[b, T - 1, h])[:, None] * np.asarray(h0, np.float64)[b, h]
            for s in range(T):
                S += (k[b, s, h] * np.exp(c[b, T - 1, h] - c[b, s, h]))[:, None] * x[b, s, h][None, :]
            hT[b, h] = S
    return o, hT


def masked_attention_shared_decay(q, f_scalar, i):
    """Literal ((Q K^T) * D) V for ONE head whose forget gate is shared by all
    key dimensions: f_scalar [T], q [T,dk], i [T,dv]; h0 = 0.

    K = 1 - f (broadcast over dk), D_ts = prod_{s<r<=t} f_r for s<=t else 0."""
    q = np.asarray(q, np.float64)
    f = np.asarray(f_scalar, np.float64)
    x = np.asarray(i, np.float64)
    T, dk = q.shape
    K = np.repeat((1.0 - f)[:, None], dk, axis=1)
    D = np.zeros((T, T))
    for t in range(T):
        for s in range(t + 1):
            D[t, s] = np.prod(f[s + 1:t + 1])
    return ((q @ K.T) * D) @ x
