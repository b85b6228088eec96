"""The float32 error metric, measured on a plain float32 implementation (no GPU).

The accuracy bar for float32 inputs is a maximum relative error of 1e-4.  An
element-wise ratio |g - r| / |r| has no bound near r = 0 for any
finite-precision arithmetic, so the metric divides by max(|r|, floor).  Which
floor a correct float32 program can meet is a property of float32 arithmetic
on this recurrence, so it is measured here, on the most direct float32 program
there is: the recurrence stepped one token at a time in PyTorch CPU float32
(with autograd for the gradients), compared with the fp64 oracle on the tiny
workload (B=1, H=2, T=64, d=16, lb=0) over ten seeds.

Recorded (worst over the seeds and over o, hT, dq, d log f, di):
  * floor 1e-3 * rms(r): about 1.9e-4, above the bar, so that floor would fail
    plain float32 itself;
  * floor 1e-3 * max|r|: about 7e-5;
  * floor 1e-2 * max|r|: about 7e-6.
The parity tests use the floor in ``parity_util.FP32_FLOOR``; this test checks
that plain float32 passes it with room to spare and that the 1e-3 * rms(r)
floor is indeed out of reach, so the choice of floor is reproducible.
"""
import numpy as np
import torch

import oracle
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import FP32_FLOOR, TOL_FP32, rel_err

SEEDS = range(1001, 1011)


def _plain_fp32(q, lf, x, dO):
    """o, hT and the gradients of <o, dO> from the token-by-token recurrence in float32."""
    q, lf, x = (t.clone().requires_grad_(True) for t in (q, lf, x))
    B, T, H, dk = q.shape
    S = torch.zeros(B, H, dk, x.shape[-1])
    outs = []
    for t in range(T):
        f = torch.exp(lf[:, t])
        k = -torch.expm1(lf[:, t])
        S = f[..., None] * S + k[..., None] * x[:, t, :, None, :]
        outs.append(torch.einsum("bhj,bhjv->bhv", q[:, t], S))
    o = torch.stack(outs, 1)
    (o * dO).sum().backward()
    return {"o": o.detach(), "hT": S.detach(), "dq": q.grad, "dlog_f": lf.grad, "di": x.grad}


def _rms_floor_err(g, r):
    g, r = np.asarray(g, np.float64), np.asarray(r, np.float64)
    return float(np.max(np.abs(g - r) / np.maximum(np.abs(r), 1e-3 * np.sqrt(np.mean(r * r)))))


def _errors():
    w = I.TINY
    worst = {"rms1e-3": 0.0, "max1e-3": 0.0, "max1e-2": 0.0, "adopted": 0.0}
    for seed in SEEDS:
        inp = I.make_inputs(w.B, w.T, w.H, w.dk, w.dv, torch.float32, w.lb, seed, with_dO=True)
        got = _plain_fp32(inp["q"], inp["log_f"], inp["i"], inp["dO"])
        n = lambda t: t.double().numpy()
        ro, rhT = oracle.fwd(n(inp["q"]), n(inp["log_f"]), n(inp["i"]))
        rdq, rdlf, rdi, _ = oracle.bwd(n(inp["q"]), n(inp["log_f"]), n(inp["i"]), n(inp["dO"]))
        ref = {"o": ro, "hT": rhT, "dq": rdq, "dlog_f": rdlf, "di": rdi}
        for name, r in ref.items():
            g = n(got[name])
            worst["rms1e-3"] = max(worst["rms1e-3"], _rms_floor_err(g, r))
            worst["max1e-3"] = max(worst["max1e-3"], rel_err(g, r, floor=1e-3))
            worst["max1e-2"] = max(worst["max1e-2"], rel_err(g, r, floor=1e-2))
            worst["adopted"] = max(worst["adopted"], rel_err(g, r))
    return worst


def test_plain_fp32_meets_the_adopted_floor_and_not_the_rms_floor():
    worst = _errors()
    print("plain float32, worst relative error by floor:", {k: f"{v:.2e}" for k, v in worst.items()},
          "adopted floor:", FP32_FLOOR)
    # the adopted floor leaves plain float32 at least a factor 1.25 below the bar
    assert worst["adopted"] <= 0.8 * TOL_FP32
    # the tighter a floor, the larger the measured error
    assert worst["max1e-2"] <= worst["max1e-3"] <= worst["rms1e-3"]
    # a floor of 1e-3 * rms(r) is beyond plain float32: it could not be the bar
    assert worst["rms1e-3"] > TOL_FP32
