"""Chunk-size invariance of the GPU routes.

The recurrence ("HGRN2: Gated Linear RNNs with State Expansion", §3.2) has no chunk length; a
chunkwise algorithm only regroups its sums.  So every supported `chunk` must give the same
results up to rounding.  The exact route (float32) really chunks by `chunk`: its results at
16, 32, 64 and 128 must agree with each other and with the oracle at the float32 bar.  The
bf16 tensor-core route always tiles by 128 tokens, so `chunk` must not change a single bit of
its results (it only sets the exact route's chunk for flagged pairs, and none is flagged here).
"""
import itertools

import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, to_cuda

pytestmark = pytest.mark.gpu

CHUNKS = (16, 32, 64, 128)


def _run(g, chunk):
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=chunk)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=chunk)
    assert L.device_status() == L.OK
    return {"o": o, "hT": hT, "dq": dq, "dlog_f": dlf, "di": di, "dh0": dh0}


def test_exact_route_results_do_not_depend_on_the_chunk(cuda):
    B, T, H, d = 2, 300, 2, 64
    inp = I.make_inputs(B, T, H, d, d, torch.float32, 0.3, seed=901, h0_sigma=0.5, with_dO=True, dhT_sigma=0.5)
    g = to_cuda(inp)
    res = {c: _run(g, c) for c in CHUNKS}
    for a, b in itertools.combinations(CHUNKS, 2):
        for name in res[a]:
            e = err(np64(res[a][name]), np64(res[b][name]), torch.float32)
            assert e <= 1e-4, (a, b, name, e)
    ref = oracle_heads(inp, [(1, 1)], want_bwd=True, dhT=inp["dhT"])
    for c in CHUNKS:
        for name, got in (("o", res[c]["o"][1, :, 1]), ("dq", res[c]["dq"][1, :, 1]),
                          ("dlog_f", res[c]["dlog_f"][1, :, 1]), ("dh0", res[c]["dh0"][1, 1])):
            assert err(np64(got), ref[name][0], torch.float32) <= 1e-4, (c, name)


def test_tensor_core_route_ignores_the_chunk_bit_for_bit(cuda):
    B, T, H = 2, 300, 4
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=902, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    res = {c: _run(g, c) for c in CHUNKS}
    L.counters(reset=True)
    _run(g, 64)
    assert L.counters(reset=True)[0] == 0   # no pair took the exact route
    for c in CHUNKS[1:]:
        for name in res[c]:
            assert torch.equal(res[c][name], res[CHUNKS[0]][name]), (c, name)
