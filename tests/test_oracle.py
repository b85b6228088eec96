"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks ``oracle`` (the C fp64 reference) against something other than
itself: a hand-worked example, an independent quadratic-form restatement, closed
forms, finite differences, or an algebraic identity.  None needs a GPU.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, B, T, H, dk, dv, lb=0.0, h0=True, scale_a=1.0):
    q = rng.standard_normal((B, T, H, dk))
    x = rng.standard_normal((B, T, H, dv))
    z = rng.standard_normal((B, T, H, dk)) * scale_a
    sig = 1.0 / (1.0 + np.exp(-z))
    log_f = np.log(lb + (1 - lb) * sig)
    h = rng.standard_normal((B, H, dk, dv)) if h0 else None
    return q, log_f, x, h


# ---------------------------------------------------------------- hand-worked example
def _parse_golden(path):
    vals = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line or "=" not in line:
            continue
        key, rhs = line.split("=", 1)
        rows = []
        for row in rhs.split(";"):
            r = []
            for tok in row.split():
                if tok.startswith("ln(") and tok.endswith(")"):
                    r.append(np.log(float(Fraction(tok[3:-1]))))
                else:
                    r.append(float(Fraction(tok)))
            rows.append(r)
        vals[key.strip()] = np.array(rows)
    return vals


def test_hand_worked_example_fwd_and_bwd():
    g = _parse_golden(os.path.join(GOLDEN, "hand_example_T2_dk2_dv2.txt"))
    sh = lambda a: a[None, :, None, :]  # [T, D] -> [1, T, 1, D]
    o, hT = oracle.fwd(sh(g["q"]), sh(g["log_f"]), sh(g["i"]))
    np.testing.assert_allclose(o[0, :, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], g["hT"], rtol=0, atol=1e-14)
    dq, dlf, di, dh0 = oracle.bwd(sh(g["q"]), sh(g["log_f"]), sh(g["i"]), sh(g["dO"]))
    np.testing.assert_allclose(dq[0, :, 0], g["dq"], atol=1e-14)
    np.testing.assert_allclose(di[0, :, 0], g["di"], atol=1e-14)
    np.testing.assert_allclose(dlf[0, :, 0], g["dlog_f"], atol=1e-14)
    np.testing.assert_allclose(dh0[0, 0], g["dh0"], atol=1e-14)


def test_scalar_decay_hand_worked_example():
    g = _parse_golden(os.path.join(GOLDEN, "hand_example_scalar_decay_T2_dk2_dv1.txt"))
    sh = lambda a: a[None, :, None, :]          # [T, D] -> [1, T, 1, D]
    lg = g["log_g"][:, 0][None, :, None]        # [T, 1] -> [1, T, 1]
    h0 = g["h0"][None, None]                    # [dk, dv] -> [1, 1, dk, dv]
    o, hT = oracle.sd_fwd(sh(g["q"]), sh(g["k"]), sh(g["v"]), lg, h0)
    np.testing.assert_allclose(o[0, :, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], g["hT"], rtol=0, atol=1e-14)
    dq, dk, dv, dlg, dh0 = oracle.sd_bwd(sh(g["q"]), sh(g["k"]), sh(g["v"]), lg, sh(g["dO"]), h0)
    np.testing.assert_allclose(dq[0, :, 0], g["dq"], atol=1e-14)
    np.testing.assert_allclose(dk[0, :, 0], g["dk"], atol=1e-14)
    np.testing.assert_allclose(dv[0, :, 0], g["dv"], atol=1e-14)
    np.testing.assert_allclose(dlg[0, :, 0], g["dlog_g"][:, 0], atol=1e-14)
    np.testing.assert_allclose(dh0[0, 0], g["dh0"], atol=1e-14)


# ---------------------------------------------------------------- forward pins
@pytest.mark.parametrize("shape", [(1, 7, 1, 3, 2), (2, 9, 3, 4, 5), (1, 70, 2, 2, 3)])
def test_fwd_matches_quadratic_form(shape):
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = shape
    q, lf, x, h0 = _rand(rng, B, T, H, dk, dv)
    o, hT = oracle.fwd(q, lf, x, h0)
    o2, hT2 = brute.quadratic_form(q, lf, x, h0)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT, hT2, rtol=1e-12, atol=1e-12)


def test_fwd_closed_form_f_one_freezes_state():
    # log f = 0 => f = 1, k = 0: S stays h0 and o_t = h0^T q_t
    rng = np.random.default_rng(2)
    q, _, x, h0 = _rand(rng, 2, 11, 2, 4, 3)
    lf = np.zeros_like(q)
    o, hT = oracle.fwd(q, lf, x, h0)
    np.testing.assert_array_equal(hT, h0)
    np.testing.assert_allclose(o, np.einsum("bthj,bhjv->bthv", q, h0), rtol=1e-13, atol=1e-13)
    o0, _ = oracle.fwd(q, lf, x, None)
    assert np.all(o0 == 0.0)


def test_fwd_closed_form_f_zero_keeps_last_input():
    # log f = -40 => f ~ 4e-18 (0 at double precision relative to 1), k = 1:
    # S_t = 1 i_t^T and o_t = (sum_j q_t[j]) i_t
    rng = np.random.default_rng(3)
    q, _, x, h0 = _rand(rng, 1, 13, 2, 5, 4)
    lf = np.full_like(q, -40.0)
    o, hT = oracle.fwd(q, lf, x, h0)
    np.testing.assert_allclose(o, q.sum(-1, keepdims=True) * x, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT[:, :, 0, :], x[:, -1], rtol=1e-12)


def test_fwd_closed_form_constant_scalar_gate_geometric_sum():
    # scalar f for all t and j, constant input xbar: S_t = f^{t+1} h0 + (1 - f^{t+1}) 1 xbar^T
    rng = np.random.default_rng(4)
    B, T, H, dk, dv = 1, 25, 1, 3, 4
    f = 0.83
    q = rng.standard_normal((B, T, H, dk))
    xbar = rng.standard_normal(dv)
    x = np.broadcast_to(xbar, (B, T, H, dv)).copy()
    h0 = rng.standard_normal((B, H, dk, dv))
    lf = np.full((B, T, H, dk), np.log(f))
    o, hT = oracle.fwd(q, lf, x, h0)
    t = np.arange(T)
    ft = f ** (t + 1)
    expect = (ft[:, None] * (q[0, :, 0] @ h0[0, 0])
              + (1 - ft)[:, None] * q[0, :, 0].sum(-1, keepdims=True) * xbar[None, :])
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT[0, 0], f ** T * h0[0, 0] + (1 - f ** T) * xbar[None, :],
                               rtol=1e-12)


def test_fwd_literal_masked_attention_when_decay_shared_over_dims():
    # with one f per token (shared across key dims) O = ((Q K^T) * D) V exactly
    rng = np.random.default_rng(5)
    T, dk, dv = 17, 4, 3
    f = 1 / (1 + np.exp(-rng.standard_normal(T)))
    q = rng.standard_normal((T, dk))
    x = rng.standard_normal((T, dv))
    lf = np.repeat(np.log(f)[:, None], dk, axis=1)
    o, _ = oracle.fwd(q[None, :, None], lf[None, :, None], x[None, :, None])
    np.testing.assert_allclose(o[0, :, 0], brute.masked_attention_shared_decay(q, f, x),
                               rtol=1e-12, atol=1e-12)


def test_fwd_heads_and_batches_independent():
    rng = np.random.default_rng(6)
    q, lf, x, h0 = _rand(rng, 2, 9, 3, 4, 4)
    o, hT = oracle.fwd(q, lf, x, h0)
    for b in range(2):
        for h in range(3):
            o1, hT1 = oracle.fwd(q[b:b + 1, :, h:h + 1], lf[b:b + 1, :, h:h + 1],
                                 x[b:b + 1, :, h:h + 1], h0[b:b + 1, h:h + 1])
            np.testing.assert_array_equal(o1[0, :, 0], o[b, :, h])
            np.testing.assert_array_equal(hT1[0, 0], hT[b, h])


# ---------------------------------------------------------------- step pins
def test_steps_equal_fwd():
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 2, 12, 3, 4, 5
    q, lf, x, h0 = _rand(rng, B, T, H, dk, dv)
    o, hT = oracle.fwd(q, lf, x, h0)
    S = h0.copy()
    for t in range(T):
        ot, S = oracle.step(q[:, t], lf[:, t], x[:, t], S)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S, hT, rtol=1e-13, atol=1e-13)


def test_step_reads_updated_state():
    # one step from S = 0 must already see the current token: o = (q . k) i
    q = np.array([[[1.0, 2.0]]])
    lf = np.log(np.array([[[0.25, 0.5]]]))
    x = np.array([[[3.0]]])
    o, S = oracle.step(q, lf, x, np.zeros((1, 1, 2, 1)))
    assert o[0, 0, 0] == pytest.approx((1 * 0.75 + 2 * 0.5) * 3.0, abs=1e-15)


# ---------------------------------------------------------------- backward pins
def _loss(q, lf, x, h0, dO, dhT):
    o, hT = oracle.fwd(q, lf, x, h0)
    return float(np.sum(o * dO) + np.sum(hT * dhT))


@pytest.mark.parametrize("T", [6, 131])
def test_bwd_matches_central_finite_differences(T):
    rng = np.random.default_rng(8 + T)
    B, H, dk, dv = 1, 2, 3, 2
    q, lf, x, h0 = _rand(rng, B, T, H, dk, dv, lb=0.3)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    dq, dlf, dx, dh0 = oracle.bwd(q, lf, x, dO, h0, dhT)
    eps = 1e-6
    pick = np.random.default_rng(99)
    for name, arr, grad in (("q", q, dq), ("log_f", lf, dlf), ("i", x, dx), ("h0", h0, dh0)):
        flat = arr.reshape(-1)
        idx = pick.choice(flat.size, size=min(flat.size, 24), replace=False)
        for n in idx:
            old = flat[n]
            flat[n] = old + eps
            lp = _loss(q, lf, x, h0, dO, dhT)
            flat[n] = old - eps
            lm = _loss(q, lf, x, h0, dO, dhT)
            flat[n] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad.reshape(-1)[n]) <= 1e-6 * max(1.0, abs(fd)), (name, n, fd)


def test_bwd_dlog_f_equals_reverse_cumsum_identity():
    # d log f_t = sum_{t'>=t} (q*dq - k*dk)_{t'} + rowsum(dhT*hT) - f_t*dk_t
    # (a rescaling argument on the cumulative log-decay; independent of BPTT's order)
    rng = np.random.default_rng(9)
    B, T, H, dk, dv = 2, 40, 2, 4, 3
    q, lf, x, h0 = _rand(rng, B, T, H, dk, dv, lb=0.2)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    dq, dlf, dx, dh0, dkk = oracle.bwd(q, lf, x, dO, h0, dhT, want_dk=True)
    _, hT = oracle.fwd(q, lf, x, h0)
    k = -np.expm1(lf)
    f = np.exp(lf)
    w = q * dq - k * dkk
    rc = np.flip(np.cumsum(np.flip(w, 1), 1), 1)
    alt = rc + np.sum(dhT * hT, -1)[:, None] - f * dkk
    np.testing.assert_allclose(dlf, alt, rtol=1e-10, atol=1e-10)


def test_bwd_linear_in_dO():
    rng = np.random.default_rng(10)
    q, lf, x, h0 = _rand(rng, 1, 15, 2, 3, 3)
    d1 = rng.standard_normal((1, 15, 2, 3))
    d2 = rng.standard_normal((1, 15, 2, 3))
    g1 = oracle.bwd(q, lf, x, d1, h0)
    g2 = oracle.bwd(q, lf, x, d2, h0)
    g12 = oracle.bwd(q, lf, x, 2 * d1 - 3 * d2, h0)
    for a, b, c in zip(g1, g2, g12):
        np.testing.assert_allclose(c, 2 * a - 3 * b, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- lower-bounded forget gate
def test_lower_bound_gate_closed_forms():
    # f = lb + (1 - lb) sigmoid(g) ("HGRN2: Gated Linear RNNs with State Expansion", §2.2)
    for lb in (0.0, 0.5, 0.9, 0.99):
        # g = 0: sigmoid = 1/2, f = (1 + lb) / 2
        assert oracle.lower_bound_log_f(0.0, lb) == pytest.approx(np.log((1 + lb) / 2), rel=1e-15, abs=1e-15)
        # g -> +inf: f -> 1 from below, 1 - f = (1 - lb) e^{-g} (1 + O(e^{-g}))
        g = 40.0
        assert -oracle.lower_bound_log_f(g, lb) == pytest.approx((1 - lb) * np.exp(-g), rel=1e-9)
        if lb > 0:   # g -> -inf: f -> lb
            assert oracle.lower_bound_log_f(-40.0, lb) == pytest.approx(np.log(lb), rel=1e-12)
    # lb = 0 is the textbook log-sigmoid: -log1p(e^{-g}) for g >= 0, g - log1p(e^{g}) for g < 0
    g = np.linspace(-20, 20, 41)
    logsig = np.where(g >= 0, -np.log1p(np.exp(-np.abs(g))), g - np.log1p(np.exp(-np.abs(g))))
    np.testing.assert_allclose(oracle.lower_bound_log_f(g, 0.0), logsig, rtol=1e-13)


def test_lower_bound_gate_matches_direct_formula_and_is_monotone():
    rng = np.random.default_rng(3)
    g = rng.normal(0, 3, 1000).clip(-10, 10)
    for lb in (0.1, 0.5, 0.95):
        direct = np.log(lb + (1 - lb) / (1 + np.exp(-g)))
        np.testing.assert_allclose(oracle.lower_bound_log_f(g, lb), direct, rtol=1e-9, atol=1e-15)
    gs = np.sort(g)
    assert np.all(np.diff(oracle.lower_bound_log_f(gs, 0.5)) >= 0)          # increasing in g
    assert np.all(oracle.lower_bound_log_f(g, 0.9) >= oracle.lower_bound_log_f(g, 0.5))   # and in lb
    assert np.all(oracle.lower_bound_log_f(g, 0.5) <= 0) and np.all(oracle.lower_bound_log_f(g, 0.5) >= np.log(0.5))


def test_lower_bound_gate_derivative_matches_finite_differences():
    # central differences of lower_bound_log_f itself, and the closed form at g = 0:
    # d log f / dg = (1 - lb) sigmoid'(0) / f(0) = (1 - lb) / 4 / ((1 + lb) / 2)
    # (for g well below 0, log f is log lb plus a tiny term, and a difference quotient of it
    # loses the digits; the tails are checked against their asymptotes instead)
    g = np.linspace(-6.0, 12.0, 73)
    h = 1e-5
    for lb in (0.0, 0.3, 0.9, 0.99):
        fd = (oracle.lower_bound_log_f(g + h, lb) - oracle.lower_bound_log_f(g - h, lb)) / (2 * h)
        np.testing.assert_allclose(oracle.lower_bound_dlog_f_dg(g, lb), fd, rtol=2e-6, atol=1e-12)
        assert oracle.lower_bound_dlog_f_dg(0.0, lb) == pytest.approx((1 - lb) / (2 * (1 + lb)), rel=1e-14)
    # far tails: e^{-g} (1 - lb) for g -> +inf; -> 0 for g -> -inf when lb > 0, -> 1 when lb = 0
    assert oracle.lower_bound_dlog_f_dg(30.0, 0.5) == pytest.approx(0.5 * np.exp(-30.0), rel=1e-6)
    assert oracle.lower_bound_dlog_f_dg(-30.0, 0.5) == pytest.approx(0.5 * np.exp(-30.0) / 0.5, rel=1e-6)
    # and it is the derivative of the log-add-exp form: sigmoid(-g) - sigmoid(log lb - g), where
    # that difference does not cancel (g >= -4)
    gg = np.linspace(-4.0, 12.0, 33)
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    for lb in (0.3, 0.9):
        np.testing.assert_allclose(oracle.lower_bound_dlog_f_dg(gg, lb), sig(-gg) - sig(np.log(lb) - gg), rtol=1e-9)
    assert oracle.lower_bound_dlog_f_dg(-30.0, 0.0) == pytest.approx(1.0, rel=1e-12)


@pytest.mark.parametrize("with_dS", [False, True])
def test_step_bwd_matches_central_finite_differences_of_step(with_dS):
    # L = <o, dO> + <S_new, dS> through oracle.step (the C decode step, not the BPTT code)
    rng = np.random.default_rng(17)
    B, H, dk, dv = 2, 1, 3, 2
    q = rng.standard_normal((B, H, dk))
    lf = -np.abs(rng.standard_normal((B, H, dk))) - 0.05
    x = rng.standard_normal((B, H, dv))
    S = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, H, dv))
    dS = rng.standard_normal((B, H, dk, dv)) if with_dS else None

    def loss(q_, lf_, x_, S_):
        o, Sn = oracle.step(q_, lf_, x_, S_)
        return float(np.sum(o * dO) + (np.sum(Sn * dS) if with_dS else 0.0))

    dq, dlf, di, dSp = oracle.step_bwd(q, lf, x, S, dO, dS)
    h = 1e-6
    for arr, grad, idx in ((q, dq, 0), (lf, dlf, 1), (x, di, 2), (S, dSp, 3)):
        fd = np.zeros_like(arr)
        for k in np.ndindex(arr.shape):
            args = [q, lf, x, S]
            p, m = arr.copy(), arr.copy()
            p[k] += h
            m[k] -= h
            args[idx] = p
            lp = loss(*args)
            args[idx] = m
            fd[k] = (lp - loss(*args)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


# ---------------------------------------------------------------- scalar-decay variant
def _sd_inputs(B, T, H, dk, dv, seed, h0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    lg = -np.abs(rng.standard_normal((B, T, H))) * 0.5
    S0 = rng.standard_normal((B, H, dk, dv)) if h0 else None
    return q, k, v, lg, S0


def test_sd_fwd_matches_quadratic_masked_form():
    # O = ((Q K^T) . D) V + Diag(prod_{r<=t} g_r) Q h0,  D_ts = prod_{s<r<=t} g_r for s <= t
    B, T, H, dk, dv = 1, 9, 2, 3, 4
    q, k, v, lg, S0 = _sd_inputs(B, T, H, dk, dv, 31)
    o, hT = oracle.sd_fwd(q, k, v, lg, S0)
    g = np.exp(lg)
    for h in range(H):
        Q, K, V = q[0, :, h], k[0, :, h], v[0, :, h]
        D = np.zeros((T, T))
        for t in range(T):
            for s in range(t + 1):
                D[t, s] = np.prod(g[0, s + 1:t + 1, h])
        G = np.array([np.prod(g[0, :t + 1, h]) for t in range(T)])
        ref = ((Q @ K.T) * D) @ V + G[:, None] * (Q @ S0[0, h])
        np.testing.assert_allclose(o[0, :, h], ref, rtol=1e-12, atol=1e-12)
        Sref = G[-1] * S0[0, h] + sum(D[T - 1, s] * np.outer(K[s], V[s]) for s in range(T))
        np.testing.assert_allclose(hT[0, h], Sref, rtol=1e-12, atol=1e-12)


def test_sd_fwd_closed_forms():
    B, T, H, dk, dv = 1, 6, 1, 3, 2
    q, k, v, _, S0 = _sd_inputs(B, T, H, dk, dv, 32)
    # g = 1: the state accumulates every k v^T on top of h0
    o, _ = oracle.sd_fwd(q, k, v, np.zeros((B, T, H)), S0)
    for t in range(T):
        S = S0[0, 0] + sum(np.outer(k[0, s, 0], v[0, s, 0]) for s in range(t + 1))
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0], rtol=1e-12, atol=1e-12)
    # g -> 0 (log g = -80): only the current token survives, o_t = (q_t . k_t) v_t
    o, _ = oracle.sd_fwd(q, k, v, np.full((B, T, H), -80.0), S0)
    np.testing.assert_allclose(o[0, :, 0], (q[0, :, 0] * k[0, :, 0]).sum(-1)[:, None] * v[0, :, 0],
                               rtol=1e-12, atol=1e-12)


def test_sd_equals_hgrn2_when_the_key_is_one_minus_a_shared_gate():
    # HGRN2 with every key dim's forget gate equal to g_t has key 1 - g_t in every dim: the
    # scalar-decay form with k_t = (1 - g_t) 1 and the same gate computes the same o and hT, and
    # the chain rule through k = 1 - g links the gradients:
    #   sum_j dlog_f[t, j] = dlog_g[t] - g_t sum_j dk[t, j]
    B, T, H, dk, dv = 2, 70, 2, 3, 4     # T crosses the oracle's 64-step checkpoint
    q, _, v, lg, S0 = _sd_inputs(B, T, H, dk, dv, 33)
    rng = np.random.default_rng(34)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    g = np.exp(lg)
    k = np.repeat((1.0 - g)[..., None], dk, axis=-1)
    lf = np.repeat(lg[..., None], dk, axis=-1)
    o1, h1 = oracle.sd_fwd(q, k, v, lg, S0)
    o2, h2 = oracle.fwd(q, lf, v, S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(h1, h2, rtol=1e-10, atol=1e-12)
    dq1, dk1, dv1, dg1, dh1 = oracle.sd_bwd(q, k, v, lg, dO, S0, dhT)
    dq2, dlf2, di2, dh2 = oracle.bwd(q, lf, v, dO, S0, dhT)
    np.testing.assert_allclose(dq1, dq2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv1, di2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dh1, dh2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dlf2.sum(-1), dg1 - g * dk1.sum(-1), rtol=1e-9, atol=1e-10)


def test_sd_bwd_matches_central_finite_differences():
    B, T, H, dk, dv = 1, 67, 1, 2, 3
    q, k, v, lg, S0 = _sd_inputs(B, T, H, dk, dv, 35)
    rng = np.random.default_rng(36)
    dO = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))

    def loss(q_, k_, v_, lg_, S_):
        o, hT = oracle.sd_fwd(q_, k_, v_, lg_, S_)
        return float(np.sum(o * dO) + np.sum(hT * dhT))

    grads = oracle.sd_bwd(q, k, v, lg, dO, S0, dhT)
    args = [q, k, v, lg, S0]
    h = 1e-6
    pick = np.random.default_rng(37)
    for ai in range(5):   # gradient ai is w.r.t. argument ai
        arr = args[ai]
        # a few entries each, including the first and the last token (a checkpoint boundary at 64)
        picks = {tuple(int(pick.integers(0, n)) for n in arr.shape) for _ in range(4)}
        if arr.ndim >= 3:
            picks |= {tuple(0 for _ in arr.shape), tuple(n - 1 for n in arr.shape)}
        for p in picks:
            a_p, a_m = arr.copy(), arr.copy()
            a_p[p] += h
            a_m[p] -= h
            ap, am = list(args), list(args)
            ap[ai], am[ai] = a_p, a_m
            fd = (loss(*ap) - loss(*am)) / (2 * h)
            assert grads[ai][p] == pytest.approx(fd, rel=1e-5, abs=1e-7), (ai, p)
