"""GPU parity of the decode-step backward (hgrn2_step_bwd, hgrn2_step_lb_bwd) against the oracle.

The oracle's step backward is the single-token case of its BPTT backward, pinned on the CPU
to finite differences of the oracle's decode step.  A chain of step backwards over T tokens is
also checked against the oracle's backward of the whole T-token recurrence.
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, tol
import oracle

pytestmark = pytest.mark.gpu

SHAPES = [
    (torch.bfloat16, 4, 3, 128, 128),
    (torch.float32, 2, 2, 16, 16),
    (torch.float32, 3, 2, 64, 32),
    (torch.bfloat16, 2, 2, 100, 12),
]


def _check(dtype, got, ref):
    dq, dlf, di, dSp = got
    rq, rlf, ri, rSp = ref
    for name, g, r in (("dq", dq, rq), ("dlog_f", dlf, rlf), ("di", di, ri)):
        e = err(np64(g), r, dtype)
        assert e <= tol(dtype), (name, e)
    if rSp is not None:   # fp32 in both dtypes: f G from fp32 arithmetic on the rounded inputs
        e = err(np64(dSp), rSp, torch.float32)
        assert e <= 1e-4, ("dS_prev", e)


@pytest.mark.parametrize("mode", ["no_dS", "dS", "in_place"])
@pytest.mark.parametrize("dtype,B,H,dk,dv", SHAPES)
def test_step_bwd_matches_oracle(cuda, dtype, B, H, dk, dv, mode):
    d = I.make_decode(B, H, dk, dv, 1, dtype, 0.8, seed=21)
    gr = I.make_step_grads(B, H, dk, dv, dtype, seed=22)
    q, lf, x, S = d["q"][0], d["log_f"][0], d["i"][0], d["S"]
    dS = None if mode == "no_dS" else gr["dS"]
    ref = oracle.step_bwd(np64(q), np64(lf), np64(x), np64(S), np64(gr["dO"]), np64(dS))
    S_dev = S.cuda()
    dS_dev = None if dS is None else dS.cuda()
    out = dS_dev if mode == "in_place" else None
    got = L.step_bwd(q.cuda(), lf.cuda(), x.cuda(), S_dev, gr["dO"].cuda(), dS_dev, dS_out=out)
    assert L.device_status() == L.OK
    if mode == "in_place":
        assert got[3].data_ptr() == dS_dev.data_ptr()
    assert torch.equal(S_dev.cpu(), S)   # the state is only read
    _check(dtype, got, ref)


@pytest.mark.parametrize("dtype,B,H,dk,dv", SHAPES[:2])
@pytest.mark.parametrize("lb", [0.0, 0.5, 0.95])
def test_step_lb_bwd_matches_oracle(cuda, dtype, B, H, dk, dv, lb):
    d = I.make_decode(B, H, dk, dv, 1, dtype, lb, seed=23)
    gr = I.make_step_grads(B, H, dk, dv, dtype, seed=24)
    q, graw, x, S = d["q"][0], d["g"][0].clone(), d["i"][0], d["S"]
    graw.view(-1)[:4] = torch.tensor([30.0, -30.0, 8.0, -8.0], dtype=dtype)   # saturated logits
    lf = oracle.lower_bound_log_f(np64(graw), lb)
    rq, rlf, ri, rSp = oracle.step_bwd(np64(q), lf, np64(x), np64(S), np64(gr["dO"]), np64(gr["dS"]))
    rg = rlf * oracle.lower_bound_dlog_f_dg(np64(graw), lb)
    got = L.step_lb_bwd(q.cuda(), graw.cuda(), x.cuda(), lb, S.cuda(), gr["dO"].cuda(), gr["dS"].cuda())
    assert L.device_status() == L.OK
    _check(dtype, got, (rq, rg, ri, rSp))


def test_step_bwd_decode_workload_full_size_sampled(cuda):
    w = I.DECODE
    d = I.make_decode(w["B"], w["H"], w["dk"], w["dv"], 1, w["dtype"], w["lb"], seed=1006)
    gr = I.make_step_grads(w["B"], w["H"], w["dk"], w["dv"], w["dtype"], seed=1007)
    dS = gr["dS"].cuda()
    got = L.step_bwd(d["q"][0].cuda(), d["log_f"][0].cuda(), d["i"][0].cuda(), d["S"].cuda(), gr["dO"].cuda(),
                     dS, dS_out=dS)
    assert L.device_status() == L.OK
    for (b, h) in [(0, 0), (17, 3), (200, 9), (255, 15)]:
        sl = lambda t: np64(t[b:b + 1, h:h + 1])
        ref = oracle.step_bwd(sl(d["q"][0]), sl(d["log_f"][0]), sl(d["i"][0]), sl(d["S"]), sl(gr["dO"]),
                              sl(gr["dS"]))
        _check(w["dtype"], tuple(t[b:b + 1, h:h + 1] for t in got), ref)


@pytest.mark.parametrize("dtype,d,T", [(torch.float32, 32, 20), (torch.bfloat16, 128, 12)])
def test_chain_of_step_backwards_equals_the_sequence_backward(cuda, dtype, d, T):
    # forward T decode steps keeping each state, then the step backwards from the last token to
    # the first with dS carried in place: dq, dlog f, di of every token and the final dS (= dh0)
    # must be the oracle's backward of the whole recurrence
    B, H = 2, 2
    inp = I.make_inputs(B, T, H, d, d, dtype, 0.7, seed=25, h0_sigma=0.3, with_dO=True, dhT_sigma=0.3)
    g = {k: v.cuda() for k, v in inp.items()}
    S = g["h0"].clone()
    states = []
    for t in range(T):
        states.append(S.clone())
        L.step(g["q"][:, t].contiguous(), g["log_f"][:, t].contiguous(), g["i"][:, t].contiguous(), S)
    dS = g["dhT"].clone()
    grads = [None] * T
    for t in reversed(range(T)):
        grads[t] = L.step_bwd(g["q"][:, t].contiguous(), g["log_f"][:, t].contiguous(), g["i"][:, t].contiguous(),
                              states[t], g["dO"][:, t].contiguous(), dS, dS_out=dS)[:3]
    assert L.device_status() == L.OK
    rq, rlf, ri, rh0 = oracle.bwd(np64(inp["q"]), np64(inp["log_f"]), np64(inp["i"]), np64(inp["dO"]),
                                  np64(inp["h0"]), np64(inp["dhT"]))
    for name, k, r in (("dq", 0, rq), ("dlog_f", 1, rlf), ("di", 2, ri)):
        got = torch.stack([grads[t][k] for t in range(T)], dim=1)
        e = err(np64(got), r, dtype)
        assert e <= tol(dtype), (name, e)
    assert err(np64(dS), rh0, dtype) <= tol(dtype)
