"""GPU parity of the d_h = 64 tensor-core route against the fp64 oracle.

bf16 heads with d_k = d_v = 64 run through the 128-wide tensor-core kernels with the second
64-column half of every operand tile held at zero ("HGRN2: Gated Linear RNNs with State
Expansion", §3.2: the head size d_h sets the state size d_h x d_h; the recurrence itself does not
depend on it).  These cases span several chunks and ragged tails, the saved-state pair, the exact
route for a flagged head, packed sequences, and the full training-sized workload (sampled).
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, to_cuda

pytestmark = pytest.mark.gpu

D = 64
CASES = [
    # B, T, H, lb, chunk, h0, dhT
    (2, 300, 2, 0.5, 64, False, False),
    (1, 300, 3, 0.95, 128, True, True),
    (1, 513, 2, 0.9, 64, True, False),
    (1, 1, 2, 0.5, 64, True, True),
    (3, 129, 4, 0.0, 64, True, True),
]


def _pairs(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


def _check(inp, got, pairs, dhT):
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=dhT)
    o, hT, dq, dlf, di, dh0 = got
    for n, (b, h) in enumerate(pairs):
        for name, g in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]),
                        ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(g), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("case", CASES)
def test_d64_fwd_bwd(cuda, case, saved):
    B, T, H, lb, chunk, with_h0, with_dhT = case
    inp = I.make_inputs(B, T, H, D, D, torch.bfloat16, lb, seed=700 + T, h0_sigma=0.1 if with_h0 else 0.0,
                        with_dO=True, dhT_sigma=0.1 if with_dhT else 0.0)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    assert (sv is not None) == saved
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g.get("h0"), want_hT=True, chunk=chunk, saved=sv)
    c = L.counters(reset=True)
    # the forward is one tensor-core launch (no sequence segments for d = 64) whatever B*H
    assert c[2] == 1 and c[1] + c[0] > 0, c
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g.get("h0"), g.get("dhT"), want_dh0=True,
                             chunk=chunk, saved=sv)
    c = L.counters(reset=True)
    # saved: one reverse-sweep launch; recompute: the forward into the workspace's saved-state
    # buffer, then that launch.  Neither touches the exact route unless a head is flagged.
    assert c[2] == (1 if saved else 2), c
    assert c[0] == 0, c   # lb = 0 included: its chunk decays are inside the factorised range
    assert L.device_status() == L.OK
    _check(inp, (o, hT, dq, dlf, di, dh0), _pairs(B, H), inp.get("dhT"))


def test_d64_strong_decay_head_takes_the_exact_route(cuda):
    B, T, H = 2, 400, 4
    inp = I.make_inputs(B, T, H, D, D, torch.bfloat16, 0.9, seed=711, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    strong = I.make_inputs(1, T, 1, D, D, torch.bfloat16, 0.0, seed=712, gate_shift=-1.0)
    inp["log_f"][1, :, 2] = strong["log_f"][0, :, 0]
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=128, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=128,
                             saved=sv)
    c = L.counters(reset=True)
    assert c[0] == 2, c   # the one flagged head, once in each pass
    assert L.device_status() == L.OK
    _check(inp, (o, hT, dq, dlf, di, dh0), [(1, 2), (0, 0), (1, 3)], inp["dhT"])


def test_d64_training_workload_full_size_sampled(cuda):
    # the training workload's hidden size with 64-wide heads: B=8, H=32, T=2048
    B, T, H = 8, 2048, 32
    inp = I.make_inputs(B, T, H, D, D, torch.bfloat16, 0.95, seed=713, with_dO=True)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    o, _ = L.fwd(g["q"], g["log_f"], g["i"], saved=sv)
    dq, dlf, di, _ = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], saved=sv)
    assert L.device_status() == L.OK
    pairs = [(0, 0), (3, 17), (7, 31)]
    ref = oracle_heads(inp, pairs, want_bwd=True)
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


def test_d64_packed_sequences(cuda):
    import oracle
    lens = [300, 0, 1, 127, 128, 129, 45]
    H = 2
    inp = I.make_varlen(lens, H, D, D, torch.bfloat16, 0.9, seed=714, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved_varlen(g["q"], g["cu_seqlens"])
    o, hT = L.fwd_varlen(g["q"], g["log_f"], g["i"], g["cu_seqlens"], g["h0"], want_hT=True, saved=sv)
    dq, dlf, di, dh0 = L.bwd_varlen(g["q"], g["log_f"], g["i"], g["dO"], g["cu_seqlens"], g["h0"], g["dhT"],
                                    want_dh0=True, saved=sv)
    assert L.device_status() == L.OK
    cu = inp["cu_seqlens"].tolist()
    for s in range(len(lens)):
        a, e = cu[s], cu[s + 1]
        for h in range(H):
            st = lambda t: np64(t[s:s + 1, h:h + 1])
            if e == a:
                assert torch.equal(hT[s, h].cpu(), inp["h0"][s, h]) and torch.equal(dh0[s, h].cpu(), inp["dhT"][s, h])
                continue
            sl = lambda t: np64(t[a:e, h:h + 1])[None]
            ro, rhT = oracle.fwd(sl(inp["q"]), sl(inp["log_f"]), sl(inp["i"]), st(inp["h0"]))
            rq, rlf, ri, rh0 = oracle.bwd(sl(inp["q"]), sl(inp["log_f"]), sl(inp["i"]), sl(inp["dO"]), st(inp["h0"]),
                                          st(inp["dhT"]))
            for name, got, r in (("o", o[a:e, h], ro[0, :, 0]), ("hT", hT[s, h], rhT[0, 0]),
                                 ("dq", dq[a:e, h], rq[0, :, 0]), ("dlog_f", dlf[a:e, h], rlf[0, :, 0]),
                                 ("di", di[a:e, h], ri[0, :, 0]), ("dh0", dh0[s, h], rh0[0, 0])):
                assert err(np64(got), r, torch.bfloat16) <= 2e-2, (name, s, h)
