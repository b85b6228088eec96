"""GPU parity of heads wider than 128 (d_k, d_v up to 256) against the fp64 oracle.

Diag(f_t) acts on each key dim alone and the update k_t i_t^T on each value column alone
("HGRN2: Gated Linear RNNs with State Expansion", §3.2 outer-product state, §5 one decay per key
dim), so a wide head runs as blocks of <= 128 whose partial outputs and gradients add.  The oracle
computes the whole wide head directly, so these cases check the split, the block routes (tensor
cores for bf16 128 x 128 and 64 x 64 blocks, the exact route otherwise), equal blocks run as extra
heads of one call, the column copies and the fp32 sums.
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, to_cuda, tol

pytestmark = pytest.mark.gpu

CASES = [
    # B, T, H, dk, dv, dtype, lb, chunk, h0, dhT
    (1, 300, 2, 256, 256, torch.bfloat16, 0.9, 64, True, True),      # four 128 x 128 tensor-core blocks, one call
    (2, 150, 1, 256, 128, torch.bfloat16, 0.9, 64, True, True),      # two 128 x 128 blocks, one call
    (2, 200, 1, 192, 192, torch.bfloat16, 0.5, 64, True, False),     # 128 x 128 and 64 x 64 tensor cores, the rest exact
    (1, 200, 2, 100, 256, torch.bfloat16, 0.9, 64, False, True),     # one key block, two value blocks (exact route)
    (2, 130, 2, 192, 160, torch.float32, 0.5, 32, True, True),       # fp32: every block on the exact route
    (1, 1, 1, 256, 256, torch.bfloat16, 0.5, 64, True, True),        # a single token
]


def _pairs(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


def _check(inp, got, pairs, dtype, dhT, names=("o", "hT", "dq", "dlog_f", "di", "dh0")):
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=dhT)
    o, hT, dq, dlf, di, dh0 = got
    for n, (b, h) in enumerate(pairs):
        cand = {"o": o[b, :, h], "hT": None if hT is None else hT[b, h], "dq": dq[b, :, h],
                "dlog_f": dlf[b, :, h], "di": di[b, :, h], "dh0": None if dh0 is None else dh0[b, h]}
        for name in names:
            e = err(np64(cand[name]), ref[name][n], dtype)
            assert e <= tol(dtype), (name, b, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[3]}x{c[4]}_{str(c[5])[6:]}_T{c[1]}" for c in CASES])
def test_wide_fwd_bwd(cuda, case, saved):
    B, T, H, dk, dv, dt, lb, chunk, with_h0, with_dhT = case
    inp = I.make_inputs(B, T, H, dk, dv, dt, lb, seed=900 + dk + dv + T, h0_sigma=0.1 if with_h0 else 0.0,
                        with_dO=True, dhT_sigma=0.1 if with_dhT else 0.0)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"], dv=dv) if saved else None
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g.get("h0"), want_hT=True, chunk=chunk, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g.get("h0"), g.get("dhT"), want_dh0=True,
                             chunk=chunk, saved=sv)
    torch.cuda.synchronize()
    assert L.device_status() == L.OK
    assert o.shape == (B, T, H, dv) and hT.shape == (B, H, dk, dv) and dq.shape == (B, T, H, dk)
    _check(inp, (o, hT, dq, dlf, di, dh0), _pairs(B, H), dt, inp.get("dhT"))


def test_wide_strong_decay_head_takes_the_exact_route(cuda):
    # one head with chunk decays past the factorised range: all four of its blocks are flagged
    # and recomputed on CUDA cores in both passes; the other head stays on the tensor cores
    B, T, H, d = 1, 300, 2, 256
    inp = I.make_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=931, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    strong = I.make_inputs(1, T, 1, d, d, torch.bfloat16, 0.0, seed=932, gate_shift=-1.0)
    inp["log_f"][0, :, 1] = strong["log_f"][0, :, 0]
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    c_fwd = L.counters(reset=True)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                             saved=sv)
    c_bwd = L.counters(reset=True)
    # the forward counts every sequence segment of a flagged block that met the bad chunk (at
    # least one per block); the backward reads the 4 flags and recomputes those blocks once
    assert c_fwd[0] >= 4 and c_bwd[0] == 4, (c_fwd, c_bwd)
    assert L.device_status() == L.OK
    _check(inp, (o, hT, dq, dlf, di, dh0), _pairs(B, H), torch.bfloat16, inp["dhT"])


def test_wide_autograd(cuda):
    B, T, H, d = 1, 260, 1, 256
    inp = I.make_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=933, with_dO=True)
    g = to_cuda(inp)
    q, lf, x = (g[k].clone().requires_grad_(True) for k in ("q", "log_f", "i"))
    o, _ = L.hgrn2(q, lf, x)
    o.backward(g["dO"])
    assert L.device_status() == L.OK
    _check(inp, (o, None, q.grad, lf.grad, x.grad, None), _pairs(B, H), torch.bfloat16, None,
           names=("o", "dq", "dlog_f", "di"))


def test_wide_training_workload_full_size_sampled(cuda):
    # the training workload's hidden size with 256-wide heads: B=8, H=8, T=2048
    B, T, H, d = 8, 2048, 8, 256
    inp = I.make_inputs(B, T, H, d, d, torch.bfloat16, 0.95, seed=934, with_dO=True)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    o, _ = L.fwd(g["q"], g["log_f"], g["i"], saved=sv)
    dq, dlf, di, _ = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], saved=sv)
    assert L.device_status() == L.OK
    pairs = [(0, 0), (5, 3), (7, 7)]
    ref = oracle_heads(inp, pairs, want_bwd=True)
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)
    assert np.isfinite(np64(o)).all()
