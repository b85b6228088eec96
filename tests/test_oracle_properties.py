"""Property-based pins of the oracle (CPU): random tiny shapes and gate strengths.

The sequential C oracle must agree with the independent explicit double-sum restatement
(oracle/brute.py) of the per-dimension recurrence ("HGRN2: Gated Linear RNNs with State
Expansion", §3.2 and §5), and its scalar-decay variant with the literal masked form
((Q K^T) . D) V, for any shape, initial state and decay strength hypothesis draws; and both
backwards must agree with central differences of their own forwards on a random entry.
"""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle
from oracle import brute

shapes = st.tuples(st.integers(1, 2), st.integers(1, 12), st.integers(1, 2), st.integers(1, 5), st.integers(1, 5))


def _draw(seed, B, T, H, dk, dv, scale):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    lf = -np.abs(rng.standard_normal((B, T, H, dk))) * scale
    x = rng.standard_normal((B, T, H, dv))
    h0 = rng.standard_normal((B, H, dk, dv))
    return q, lf, x, h0


@settings(max_examples=40, deadline=None)
@given(shape=shapes, seed=st.integers(0, 10 ** 6), scale=st.sampled_from([0.01, 0.3, 2.0, 20.0]),
       with_h0=st.booleans())
def test_fwd_equals_explicit_double_sum(shape, seed, scale, with_h0):
    B, T, H, dk, dv = shape
    q, lf, x, h0 = _draw(seed, B, T, H, dk, dv, scale)
    h0 = h0 if with_h0 else None
    o, hT = oracle.fwd(q, lf, x, h0)
    o2, hT2 = brute.quadratic_form(q, lf, x, h0)
    np.testing.assert_allclose(o, o2, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(hT, hT2, rtol=1e-9, atol=1e-11)


@settings(max_examples=40, deadline=None)
@given(shape=shapes, seed=st.integers(0, 10 ** 6), scale=st.sampled_from([0.01, 0.3, 2.0, 20.0]))
def test_sd_fwd_equals_literal_masked_form(shape, seed, scale):
    B, T, H, dk, dv = shape
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    lg = -np.abs(rng.standard_normal((B, T, H))) * scale
    o, _ = oracle.sd_fwd(q, k, v, lg)
    g = np.exp(lg)
    for b in range(B):
        for h in range(H):
            D = np.zeros((T, T))
            for t in range(T):
                for s in range(t + 1):
                    D[t, s] = np.prod(g[b, s + 1:t + 1, h])
            ref = ((q[b, :, h] @ k[b, :, h].T) * D) @ v[b, :, h]
            np.testing.assert_allclose(o[b, :, h], ref, rtol=1e-9, atol=1e-11)


@settings(max_examples=25, deadline=None)
@given(shape=shapes, seed=st.integers(0, 10 ** 6), scale=st.sampled_from([0.05, 0.5, 3.0]),
       which=st.integers(0, 3))
def test_bwd_matches_central_difference_on_a_random_entry(shape, seed, scale, which):
    B, T, H, dk, dv = shape
    q, lf, x, h0 = _draw(seed, B, T, H, dk, dv, scale)
    rng = np.random.default_rng(seed + 1)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    args = [q, lf, x, h0]

    def loss(a):
        o, hT = oracle.fwd(*a)
        return float(np.sum(o * dO) + np.sum(hT * dhT))

    grads = oracle.bwd(q, lf, x, dO, h0, dhT)   # dq, dlog_f, di, dh0 <-> q, log_f, i, h0
    arr = args[which]
    idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
    h = 1e-6
    ap, am = [a.copy() for a in args], [a.copy() for a in args]
    ap[which][idx] += h
    am[which][idx] -= h
    fd = (loss(ap) - loss(am)) / (2 * h)
    assert grads[which][idx] == pytest.approx(fd, rel=1e-5, abs=1e-6)


@settings(max_examples=25, deadline=None)
@given(B=st.integers(1, 2), T=st.integers(1, 9), H=st.integers(1, 2), dk=st.integers(2, 6), dv=st.integers(2, 6),
       seed=st.integers(0, 10 ** 6), scale=st.sampled_from([0.05, 0.5, 3.0]), data=st.data())
def test_blocks_of_key_and_value_dims_recombine_exactly(B, T, H, dk, dv, seed, scale, data):
    # Diag(f) acts on each key dim and the update on each value column alone (§3.2, §5), so the
    # state block S[a, c] of key block a and value block c is a recurrence of its own: o[c] sums
    # the blocks' outputs over a, dq and d log f [a] sum over c, di[c] over a, and hT, dh0 blocks
    # map one to one.  Heads wider than 128 run on exactly this split.
    ka = data.draw(st.integers(1, dk - 1))
    vc = data.draw(st.integers(1, dv - 1))
    q, lf, x, h0 = _draw(seed, B, T, H, dk, dv, scale)
    rng = np.random.default_rng(seed + 2)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    o, hT = oracle.fwd(q, lf, x, h0)
    dq, dlf, di, dh0 = oracle.bwd(q, lf, x, dO, h0, dhT)
    K = [slice(0, ka), slice(ka, dk)]
    V = [slice(0, vc), slice(vc, dv)]
    o2, hT2 = np.zeros_like(o), np.zeros_like(hT)
    dq2, dlf2, di2, dh02 = np.zeros_like(dq), np.zeros_like(dlf), np.zeros_like(di), np.zeros_like(dh0)
    for a in K:
        for c in V:
            ob, hb = oracle.fwd(q[..., a], lf[..., a], x[..., c], h0[:, :, a, c])
            o2[..., c] += ob
            hT2[:, :, a, c] = hb
            gq, gf, gi, gh = oracle.bwd(q[..., a], lf[..., a], x[..., c], dO[..., c], h0[:, :, a, c], dhT[:, :, a, c])
            dq2[..., a] += gq
            dlf2[..., a] += gf
            di2[..., c] += gi
            dh02[:, :, a, c] = gh
    for got, ref in ((o2, o), (hT2, hT), (dq2, dq), (dlf2, dlf), (di2, di), (dh02, dh0)):
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)
