"""Sequence parallelism on the GPU: the slice state maps, their scan, and whole sequences split
into slices ("ranks") run one after the other on one device, against the oracle.

The ranks are emulated in one process through the driver's phases (every rank's local maps,
then every rank's finish with the stacked maps): no kernel waits on another, and the same
kernels run as on several GPUs.  The exchange across a real process group is covered on CPU by
test_seqpar_ranks.py.
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from linear_attention_hgrn2_b200 import seqpar
from parity_util import err, np64, oracle_heads, tol
import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,B,T,H,dk,dv,lb", [
    (torch.float32, 2, 77, 3, 16, 24, 0.0),
    (torch.float32, 1, 300, 2, 128, 128, 0.5),
    (torch.bfloat16, 2, 300, 3, 128, 128, 0.9),     # forward map on the tensor cores
    (torch.bfloat16, 1, 1000, 2, 128, 128, 0.0),    # ... at lb = 0
    (torch.bfloat16, 2, 200, 2, 64, 64, 0.5),
    (torch.bfloat16, 1, 150, 2, 100, 200, 0.5),     # dv > 128: value columns in blocks of 32
    (torch.float32, 1, 0, 2, 16, 16, 0.5),          # an empty slice: g = 1, U = W = 0
])
def test_state_maps_match_the_oracle(cuda, dtype, B, T, H, dk, dv, lb):
    inp = I.make_inputs(B, T, H, dk, dv, dtype, lb, seed=800 + T + dk, with_dO=True)
    g_, U = L.state_map(inp["log_f"].cuda(), inp["i"].cuda())
    g2, W = L.state_map_bwd(inp["q"].cuda(), inp["log_f"].cuda(), inp["dO"].cuda())
    torch.cuda.synchronize()
    lf = np64(inp["log_f"])
    g_ref = np.exp(lf.sum(axis=1))
    if T == 0:
        assert torch.all(g_ == 1) and torch.all(U == 0) and torch.all(W == 0)
        return
    _, U_ref = oracle.fwd(np.zeros_like(lf), lf, np64(inp["i"]))
    W_ref = oracle.bwd(np64(inp["q"]), lf, np.zeros_like(np64(inp["dO"])), np64(inp["dO"]))[3]
    # g: a product of T gates in fp32, held to the fp32 bar whatever the input dtype
    assert err(np64(g_), g_ref, torch.float32) <= 1e-4
    assert err(np64(g2), g_ref, torch.float32) <= 1e-4
    assert err(np64(U), U_ref, dtype) <= tol(dtype)
    assert err(np64(W), W_ref, dtype) <= tol(dtype)


def test_affine_scan_matches_a_plain_loop(cuda):
    R, B, H, dk, dv = 5, 2, 3, 16, 8
    gen = torch.Generator().manual_seed(3)
    g = torch.rand((R, B, H, dk), generator=gen)
    M = torch.randn((R, B, H, dk, dv), generator=gen)
    init = torch.randn((B, H, dk, dv), generator=gen)

    def plain(first, count, step, S0):
        S = S0.double().clone()
        r = first
        for _ in range(count):
            S = g[r].double()[..., None] * S + M[r].double()
            r += step
        return S.numpy()

    gc, Mc, ic = g.cuda(), M.cuda(), init.cuda()
    for first, count, step in ((0, 3, 1), (0, 5, 1), (4, 2, -1), (4, 5, -1), (2, 0, 1)):
        S = L.affine_scan(gc, Mc, first, count, step, init=ic)
        assert err(np64(S), plain(first, count, step, init), torch.float32) <= 1e-5
    S0 = L.affine_scan(gc, Mc, 0, 5, 1)            # no init: zeros
    assert err(np64(S0), plain(0, 5, 1, torch.zeros_like(init)), torch.float32) <= 1e-5
    inplace = ic.clone()
    L.affine_scan(gc, Mc, 1, 3, 1, init=inplace, out=inplace)
    assert err(np64(inplace), plain(1, 3, 1, init), torch.float32) <= 1e-5
    with pytest.raises(L.HGRN2Error):
        L.affine_scan(gc, Mc, 3, 3, 1)             # maps 3, 4, 5: past R


def _emulate(inp, bounds, saved, backward=True):
    """Every slice's local maps, then every slice's finish, in one process (ranks in turn)."""
    R = len(bounds) - 1
    sl = [{k: inp[k][:, bounds[r]:bounds[r + 1]].contiguous()
           for k in ("q", "log_f", "i", "dO") if k in inp} for r in range(R)]
    maps = [seqpar.fwd_local(s["q"], s["log_f"], s["i"]) for s in sl]
    g_all = torch.stack([m[0] for m in maps])
    U_all = torch.stack([m[1] for m in maps])
    fw = []
    for r, s in enumerate(sl):
        sv = L.new_saved(s["q"]) if saved else None
        o, hT, ctx = seqpar.fwd_finish(s["q"], s["log_f"], s["i"], g_all, U_all, r, inp.get("h0"), saved=sv)
        fw.append((o, hT, ctx, sv))
    out = {"o": torch.cat([f[0] for f in fw], 1), "hT": [f[1] for f in fw]}
    if backward:
        W_all = torch.stack([seqpar.bwd_local(s["q"], s["log_f"], s["dO"]) for s in sl])
        gr = [seqpar.bwd_finish(s["q"], s["log_f"], s["i"], s["dO"], fw[r][2], W_all, inp.get("dhT"), saved=fw[r][3])
              for r, s in enumerate(sl)]
        for n, name in enumerate(("dq", "dlog_f", "di")):
            out[name] = torch.cat([x[n] for x in gr], 1)
        out["dh0"] = gr[0][3]
        assert all(x[3] is None for x in gr[1:])
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("R", [2, 4])
def test_long_workload_split_across_ranks(cuda, R):
    # the long-sequence workload (B=1, H=8, T=32768, lb=0.9, h0 ~ N(0, 0.1^2), hT returned),
    # one contiguous slice per rank
    w = I.LONG
    inp = I.make_workload(w, seed=1004)
    g = {k: v.cuda() for k, v in inp.items()}
    bounds = np.linspace(0, w.T, R + 1).astype(int)
    out = _emulate(g, bounds, saved=False, backward=False)
    assert L.device_status() == L.OK
    pairs = [(0, 0), (0, 5)]
    ref = oracle_heads(inp, pairs)
    for n, (b, h) in enumerate(pairs):
        assert err(np64(out["o"][b, :, h]), ref["o"][n], w.dtype) <= tol(w.dtype)
        for hT in out["hT"]:   # every rank holds the whole sequence's final state
            assert err(np64(hT[b, h]), ref["hT"][n], w.dtype) <= tol(w.dtype)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("dtype,lb,bounds", [
    (torch.bfloat16, 0.5, [0, 250, 600, 700]),   # three ranks, unequal slices, ragged chunks
    (torch.bfloat16, 0.0, [0, 384, 768]),        # lb = 0 across two ranks
    (torch.float32, 0.9, [0, 100, 130, 300]),
])
def test_fwd_bwd_split_across_ranks(cuda, saved, dtype, lb, bounds):
    B, H, d = 2, 3, 128
    T = bounds[-1]
    inp = I.make_inputs(B, T, H, d, d, dtype, lb, seed=900 + T, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    out = _emulate({k: v.cuda() for k, v in inp.items()}, bounds, saved=saved and dtype == torch.bfloat16)
    assert L.device_status() == L.OK
    pairs = [(b, h) for b in range(B) for h in range(H)]
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", out["o"][b, :, h]), ("hT", out["hT"][-1][b, h]), ("dq", out["dq"][b, :, h]),
                          ("dlog_f", out["dlog_f"][b, :, h]), ("di", out["di"][b, :, h]),
                          ("dh0", out["dh0"][b, h])):
            e = err(np64(got), ref[name][n], dtype)
            assert e <= tol(dtype), (name, b, h, e)
