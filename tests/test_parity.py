"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Element-by-element comparisons on identical seeded inputs: small sizes that
span several chunks and a ragged tail (whole tensors compared), and the full
workload sizes in the launch configuration the benchmark times (sampled
(batch, head) pairs, each an independent problem, compared whole).
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, to_cuda, tol
import oracle

pytestmark = pytest.mark.gpu


def _check_fwd(inp, o, hT, pairs, dtype):
    ref = oracle_heads(inp, pairs)
    for n, (b, h) in enumerate(pairs):
        e = err(np64(o[b, :, h]), ref["o"][n], dtype)
        assert e <= tol(dtype), ("o", b, h, e)
        if hT is not None:
            e = err(np64(hT[b, h]), ref["hT"][n], dtype)
            assert e <= tol(dtype), ("hT", b, h, e)


def _all_pairs(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


# ---------------------------------------------------------------- tiny workload (fp32, chunk 16)
def test_tiny_workload_fwd(cuda):
    w = I.TINY
    inp = to_cuda(I.make_workload(w, seed=1001))
    o, hT = L.fwd(inp["q"], inp["log_f"], inp["i"], want_hT=True, chunk=w.chunk)
    _check_fwd(inp, o, hT, _all_pairs(w.B, w.H), w.dtype)


# ---------------------------------------------------------------- fp32, exact route, whole tensors
FP32_CASES = [
    # B, T, H, dk, dv, chunk
    (1, 64, 2, 16, 16, 16),
    (2, 100, 3, 32, 16, 32),
    (1, 77, 2, 64, 48, 64),
    (1, 150, 1, 128, 128, 32),
    (1, 45, 2, 128, 128, 128),
    (3, 1, 2, 8, 4, 16),
]


@pytest.mark.parametrize("case", FP32_CASES)
def test_fp32_fwd_bwd(cuda, case):
    B, T, H, dk, dv, chunk = case
    inp = I.make_inputs(B, T, H, dk, dv, torch.float32, 0.0, seed=7 + T, h0_sigma=0.5, with_dO=True,
                        dhT_sigma=0.5)
    g = to_cuda(inp)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=chunk)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True,
                             chunk=chunk)
    ref = oracle_heads(inp, _all_pairs(B, H), want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(_all_pairs(B, H)):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]),
                          ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], torch.float32)
            assert e <= 1e-4, (name, b, h, e)


# ---------------------------------------------------------------- bf16, d = 128, whole tensors
BF16_CASES = [
    # B, T, H, lb, chunk, h0, dhT
    (2, 300, 2, 0.5, 64, False, False),
    (1, 300, 3, 0.95, 128, True, True),
    (1, 513, 2, 0.9, 64, True, False),
    (2, 129, 1, 0.0, 128, False, True),
    (1, 1, 2, 0.5, 64, True, True),
]


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("case", BF16_CASES)
def test_bf16_fwd_bwd(cuda, case, saved):
    B, T, H, lb, chunk, with_h0, with_dhT = case
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, lb, seed=100 + T,
                        h0_sigma=0.1 if with_h0 else 0.0, with_dO=True,
                        dhT_sigma=0.1 if with_dhT else 0.0)
    g = to_cuda(inp)
    h0, dhT = g.get("h0"), g.get("dhT")
    sv = L.new_saved(g["q"]) if saved else None
    assert (sv is not None) == saved
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], h0, want_hT=True, chunk=chunk, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], h0, dhT, want_dh0=True, chunk=chunk,
                             saved=sv)
    ref = oracle_heads(inp, _all_pairs(B, H), want_bwd=True, dhT=inp.get("dhT"))
    for n, (b, h) in enumerate(_all_pairs(B, H)):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]),
                          ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


# ---------------------------------------------------------------- full workload sizes, sampled heads
def _sample_pairs(B, H, n, seed):
    rng = np.random.default_rng(seed)
    allp = _all_pairs(B, H)
    idx = rng.choice(len(allp), size=min(n, len(allp)), replace=False)
    return sorted({allp[i] for i in idx} | {allp[0], allp[-1]})


def test_workload_fwd_layer_full_size(cuda):
    w = I.FWD_LAYER
    inp = I.make_workload(w, seed=1002)
    g = to_cuda(inp)
    o, _ = L.fwd(g["q"], g["log_f"], g["i"], chunk=w.chunk)
    torch.cuda.synchronize()
    _check_fwd(inp, o, None, _sample_pairs(w.B, w.H, 4, 1), w.dtype)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_workload_train_full_size_fwd_bwd(cuda, saved):
    # saved=True is the pair the benchmark times: hgrn2_fwd_train + hgrn2_bwd_saved
    w = I.TRAIN
    inp = I.make_workload(w, seed=1003)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    o, _ = L.fwd(g["q"], g["log_f"], g["i"], chunk=w.chunk, saved=sv)
    dq, dlf, di, _ = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], chunk=w.chunk, saved=sv)
    torch.cuda.synchronize()
    pairs = _sample_pairs(w.B, w.H, 3, 2)
    ref = oracle_heads(inp, pairs, want_bwd=True)
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]),
                          ("di", di[b, :, h])):
            e = err(np64(got), ref[name][n], w.dtype)
            assert e <= 2e-2, (name, b, h, e)


def test_workload_long_full_size_with_h0_hT(cuda):
    w = I.LONG
    inp = I.make_workload(w, seed=1004)
    g = to_cuda(inp)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=w.chunk)
    torch.cuda.synchronize()
    _check_fwd(inp, o, hT, [(0, 0), (0, 5)], w.dtype)


# ---------------------------------------------------------------- edge cases and degenerate gates
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_T_zero_copies_state(cuda, dtype):
    h0 = torch.randn(2, 3, 128, 128, device="cuda")
    q = torch.empty(2, 0, 3, 128, device="cuda", dtype=dtype)
    o, hT = L.fwd(q, q, q, h0, want_hT=True)
    assert o.numel() == 0
    assert torch.equal(hT, h0)
    dq, dlf, di, dh0 = L.bwd(q, q, q, q, h0, h0 * 2, want_dh0=True)
    assert torch.equal(dh0, h0 * 2)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_one_freezes_state(cuda, dtype):
    # log f = 0: f = 1, k = 0 => S stays h0 and o_t = h0^T q_t
    B, T, H, d = 1, 200, 2, 128
    q = torch.randn(B, T, H, d).to(dtype)
    h0 = torch.randn(B, H, d, d) * 0.1
    x = torch.randn(B, T, H, d).to(dtype)
    lf = torch.zeros(B, T, H, d, dtype=dtype)
    o, hT = L.fwd(q.cuda(), lf.cuda(), x.cuda(), h0.cuda(), want_hT=True, chunk=64)
    ref = torch.einsum("bthj,bhjv->bthv", q.double(), h0.double())
    assert err(np64(o), ref.numpy(), dtype) <= tol(dtype)
    assert torch.allclose(hT.cpu(), h0, atol=0, rtol=0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_zero_keeps_last_input(cuda, dtype):
    # log f = -40 (f ~ 4e-18): o_t = (sum_j q_t[j]) i_t ; every chunk's decay span is huge
    B, T, H, d = 1, 257, 2, 128
    q = torch.randn(B, T, H, d).to(dtype)
    x = torch.randn(B, T, H, d).to(dtype)
    lf = torch.full((B, T, H, d), -40.0).to(dtype)
    dO = torch.randn(B, T, H, d).to(dtype)
    g = [t.cuda() for t in (q, lf, x, dO)]
    o, hT = L.fwd(g[0], g[1], g[2], want_hT=True, chunk=128)
    ref = (q.double().sum(-1, keepdim=True) * x.double()).numpy()
    assert np.isfinite(np64(o)).all()
    assert err(np64(o), ref, dtype) <= tol(dtype)
    dq, dlf, di, _ = L.bwd(*g, chunk=128)
    r = oracle.bwd(np64(q), np64(lf), np64(x), np64(dO))
    for got, want in zip((dq, di), (r[0], r[2])):
        assert np.isfinite(np64(got)).all()
        assert err(np64(got), want, dtype) <= tol(dtype)
    # d log f is ~1e-17 here (every path through f carries a factor f).  The chunkwise
    # backward forms it as a reverse cumulative sum of q*dq - k*dk, whose summands are O(1)
    # and cancel; its error is therefore bounded against the scale of those summands.
    scale = np.max(np.abs(np64(q) * r[0]))
    assert np.isfinite(np64(dlf)).all()
    assert np.max(np.abs(np64(dlf) - r[1])) <= tol(dtype) * scale


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_lower_bound_zero_stays_on_tensor_cores(cuda, saved):
    # lb = 0 (the first layer's bound) at chunk 128: cumulative log-decay spans of about -103
    # inside a chunk.  The balanced reference keeps every factor within e^{+-75}, so no pair
    # leaves the tensor cores (B*H = 2: the forward runs in sequence segments)
    inp = I.make_inputs(1, 384, 2, 128, 128, torch.bfloat16, 0.0, seed=5, with_dO=True)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    L.counters(reset=True)
    o, _ = L.fwd(g["q"], g["log_f"], g["i"], chunk=128, saved=sv)
    dq, dlf, di, _ = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], chunk=128, saved=sv)
    c = L.counters(reset=True)
    assert c[0] == 0, c   # no exact-route pass
    assert L.device_status() == L.OK
    ref = oracle_heads(inp, [(0, 0), (0, 1)], want_bwd=True)
    for n, h in enumerate((0, 1)):
        for name, got in (("o", o[0, :, h]), ("dq", dq[0, :, h]), ("dlog_f", dlf[0, :, h]),
                          ("di", di[0, :, h])):
            assert np.isfinite(np64(got)).all()
            assert err(np64(got), ref[name][n], torch.bfloat16) <= 2e-2, name


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_workload_train_lower_bound_zero_full_size(cuda, saved):
    # the training workload's shape with the first layer's lower bound, lb = 0 (forget gates
    # sigmoid(x), x ~ N(0, 1)), in the launch configuration the benchmark times: every pair on
    # the tensor cores, sampled pairs checked whole against the oracle
    w = I.TRAIN
    inp = I.make_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, 0.0, seed=1013, with_dO=True, h0_sigma=0.1,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=w.chunk, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True,
                             chunk=w.chunk, saved=sv)
    c = L.counters(reset=True)
    assert c[0] == 0, c
    assert L.device_status() == L.OK
    pairs = _sample_pairs(w.B, w.H, 3, 3)
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]),
                          ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], w.dtype)
            assert e <= 2e-2, (name, b, h, e)


def test_saved_pair_launch_counts_and_mixed_routes(cuda):
    # B*H = 80 > 148 / 2: one CTA per (b,h), no sequence segments.  Head 3 of batch 1 gets
    # gates shifted down (chunk decays of ~-180, past the factorised range: exact route), every other
    # pair stays on the tensor cores; the saved backward is one launch and computes both kinds
    # of pair.
    B, T, H = 10, 600, 8
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=77, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    strong = I.make_inputs(1, T, 1, 128, 128, torch.bfloat16, 0.0, seed=78, gate_shift=-1.0)
    inp["log_f"][1, :, 3] = strong["log_f"][0, :, 0]
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    c_fwd = L.counters(reset=True)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                             saved=sv)
    c_bwd = L.counters(reset=True)
    assert c_fwd[2] == 1 and c_bwd[2] == 1, (c_fwd, c_bwd)
    assert c_fwd[0] == 1 and c_bwd[0] == 1, (c_fwd, c_bwd)   # one exact-route pair in each pass
    assert L.device_status() == L.OK
    pairs = [(1, 3), (0, 0), (1, 7)]
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]),
                          ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


def test_autograd_function_uses_saved_states(cuda):
    B, T, H = 1, 260, 2
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.95, seed=9, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    q, lf, x = (g[k].clone().requires_grad_(True) for k in ("q", "log_f", "i"))
    h0 = g["h0"].clone().requires_grad_(True)
    L.counters(reset=True)
    o, hT = L.hgrn2(q, lf, x, h0, chunk=64)
    loss = (o.float() * g["dO"].float()).sum() + (hT * g["dhT"]).sum()
    loss.backward()
    c = L.counters(reset=True)
    # segmented forward (3 segments per pair: segments, then the fix-up that sums the entering states
    # itself) + segmented saved backward (segments, then the fix-up that sums the carried gradients
    # itself)
    assert c[2] == 2 + 2, c
    ref = oracle_heads(inp, [(0, 0), (0, 1)], want_bwd=True, dhT=inp["dhT"])
    for n, h in enumerate((0, 1)):
        for name, got in (("dq", q.grad[0, :, h]), ("dlog_f", lf.grad[0, :, h]), ("di", x.grad[0, :, h]),
                          ("dh0", h0.grad[0, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_more_pairs_than_sms(cuda, saved):
    # B*H = 192 > 148 SMs: the one-CTA-per-(b,h) kernels run in more than one wave; ragged T
    B, T, H = 2, 200, 96
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=31, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                             saved=sv)
    assert L.device_status() == L.OK
    pairs = [(0, 0), (0, 95), (1, 0), (1, 47), (1, 95)]
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]),
                          ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["plain", "saved"])
def test_segmented_forward_with_a_flagged_pair(cuda, saved):
    # B*H = 2: the forward runs in 8 sequence segments (segments, then the fix-up, which sums the
    # states entering them itself: 2 launches).  Head 1
    # has gates shifted below the factorised range: its segments flag it, and the last of its
    # segments to finish recomputes the whole sequence on the exact route in the same launch
    B, T, H = 1, 1000, 2
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=61, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    strong = I.make_inputs(1, T, 1, 128, 128, torch.bfloat16, 0.0, seed=62, gate_shift=-1.0)
    inp["log_f"][0, :, 1] = strong["log_f"][0, :, 0]
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    c = L.counters(reset=True)
    assert c[2] == 2 and c[0] >= 1, c
    assert L.device_status() == L.OK
    want_bwd = saved
    if saved:
        dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                                 saved=sv)
    ref = oracle_heads(inp, [(0, 0), (0, 1)], want_bwd=want_bwd, dhT=inp["dhT"])
    for n, h in enumerate((0, 1)):
        got = [("o", o[0, :, h]), ("hT", hT[0, h])]
        if saved:
            got += [("dq", dq[0, :, h]), ("dlog_f", dlf[0, :, h]), ("di", di[0, :, h]), ("dh0", dh0[0, h])]
        for name, t in got:
            e = err(np64(t), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["plain", "saved"])
@pytest.mark.parametrize("lb", [0.9, 0.5])
def test_segmented_forward_few_segments(cuda, saved, lb):
    # B*H = 40: 3 segments of 3 chunks per pair (ragged T), so the fix-up sums the entering states
    # itself and writes hT (2 launches).  At lb = 0.9 the carried state matters through whole
    # segments (the fix-up walks every chunk of them, from one or two stages); at 0.5 for one chunk.
    # Head 7 of batch 1 has gates below the factorised range and is recomputed on the exact route.
    B, T, H = 2, 1000, 20
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, lb, seed=63, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    strong = I.make_inputs(1, T, 1, 128, 128, torch.bfloat16, 0.0, seed=64, gate_shift=-1.0)
    inp["log_f"][1, :, 7] = strong["log_f"][0, :, 0]
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    c = L.counters(reset=True)
    assert c[2] == 2 and c[0] >= 1, c
    assert L.device_status() == L.OK
    if saved:
        dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                                 saved=sv)
    pairs = [(0, 0), (0, 19), (1, 6), (1, 7), (1, 19)]
    ref = oracle_heads(inp, pairs, want_bwd=saved, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        got = [("o", o[b, :, h]), ("hT", hT[b, h])]
        if saved:
            got += [("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h]), ("dh0", dh0[b, h])]
        for name, t in got:
            e = err(np64(t), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


@pytest.mark.parametrize("saved", [False, True], ids=["plain", "saved"])
@pytest.mark.parametrize("lb", [0.999, 0.9])
def test_segmented_forward_walks_back_as_far_as_the_states_matter(cuda, saved, lb):
    # B*H = 8, T = 2304: 18 one-chunk segments per pair.  The fix-up of segment k sums the maps of
    # segments k-1, k-2, ... while what the rest could add is at least 2^-24: at lb = 0.999 (a
    # chunk keeps ~94% of the state) that is every earlier segment, and the last segment's hT sums
    # all 17; at lb = 0.9 a few.  Checked against the oracle with h0 and hT, and (saved) through
    # the corrected chunk states that the backward reads.
    B, T, H = 1, 2304, 8
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, lb, seed=1170 + int(lb * 1000), h0_sigma=0.1,
                        with_dO=True, dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    c = L.counters(reset=True)
    assert c[2] == 2 and c[0] == 0, c
    assert L.device_status() == L.OK
    if saved:
        dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                                 saved=sv)
    pairs = [(0, 0), (0, 3), (0, 7)]
    ref = oracle_heads(inp, pairs, want_bwd=saved, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        got = [("o", o[b, :, h]), ("hT", hT[b, h])]
        if saved:
            got += [("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]), ("di", di[b, :, h]), ("dh0", dh0[b, h])]
        for name, t in got:
            e = err(np64(t), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


@pytest.mark.parametrize("saved", [True, False], ids=["saved", "recompute"])
@pytest.mark.parametrize("lb,T", [(0.9, 32768), (0.0, 4096)])
def test_segmented_backward_long_sequence(cuda, lb, T, saved):
    # B*H = 8, the long workload's shape as a training pair: the saved-state backward runs in
    # segments (18 of 15 chunks per pair at T = 32768; 16 of 2 at T = 4096): every segment's reverse
    # sweep from a zero gradient (the last from dhT), then the carried gradients, summed from the
    # later segments' maps, added to di and d log f of each segment's last chunks (and dh0).
    # Without saved states the backward first runs the training forward into its workspace (2 more
    # launches).  lb = 0: strong decay.
    B, H = 1, 8
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, lb, seed=1090 + T, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"]) if saved else None
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    L.counters(reset=True)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                             saved=sv)
    c = L.counters(reset=True)
    assert c[2] == (2 if saved else 4) and c[0] == 0, c
    assert L.device_status() == L.OK
    pairs = [(0, 0), (0, 5)]
    ref = oracle_heads(inp, pairs, want_bwd=True, dhT=inp["dhT"])
    for n, (b, h) in enumerate(pairs):
        for name, got in (("o", o[b, :, h]), ("hT", hT[b, h]), ("dq", dq[b, :, h]), ("dlog_f", dlf[b, :, h]),
                          ("di", di[b, :, h]), ("dh0", dh0[b, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, b, h, e)


def test_saved_pair_long_segmented_sequence(cuda):
    # B*H = 2: the forward cuts each sequence into 32 one-chunk segments (segments from zero states,
    # fp32 scan, carried-state fix-up) and saves the chunk states of all of them; the backward runs
    # the same 32 segments (reverse sweeps, reverse fp32 scan of their maps, carried-gradient
    # fix-up).  More than 18 segments per pair: both scans are launches of their own.
    B, T, H = 1, 4096, 2
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.95, seed=41, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    L.counters(reset=True)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
    assert L.counters(reset=True)[2] == 3
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64,
                             saved=sv)
    assert L.counters(reset=True)[2] == 3
    assert L.device_status() == L.OK
    ref = oracle_heads(inp, [(0, 0), (0, 1)], want_bwd=True, dhT=inp["dhT"])
    for n, h in enumerate((0, 1)):
        for name, got in (("o", o[0, :, h]), ("hT", hT[0, h]), ("dq", dq[0, :, h]), ("dlog_f", dlf[0, :, h]),
                          ("di", di[0, :, h]), ("dh0", dh0[0, h])):
            e = err(np64(got), ref[name][n], torch.bfloat16)
            assert e <= 2e-2, (name, h, e)


def test_calls_on_a_side_stream(cuda):
    # every call is asynchronous on torch's current stream; results on a side stream match the
    # default stream's bit for bit
    inp = I.make_inputs(2, 300, 4, 128, 128, torch.bfloat16, 0.9, seed=51, with_dO=True)
    g = to_cuda(inp)
    sv0 = L.new_saved(g["q"])
    o0, _ = L.fwd(g["q"], g["log_f"], g["i"], chunk=64, saved=sv0)
    r0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], chunk=64, saved=sv0)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        sv1 = L.new_saved(g["q"])
        o1, _ = L.fwd(g["q"], g["log_f"], g["i"], chunk=64, saved=sv1)
        r1 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], chunk=64, saved=sv1)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1)
    for a, b in zip(r0[:3], r1[:3]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,T,H", [(2, 300, 3), (4, 260, 20)], ids=["segments", "pair_per_cta"])
def test_cuda_graph_capture_replays_bit_for_bit(cuda, B, T, H):
    # the training pair captured into a CUDA graph (its memsets, launches and programmatic
    # dependent launches are all stream-ordered) and replayed on new inputs copied into the
    # captured buffers: the replay equals eager calls on those inputs bit for bit.  B*H = 6 runs
    # both calls in sequence segments; B*H = 80 one CTA per (b,h).
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=71, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    inp2 = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.9, seed=72, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    g = to_cuda(inp)
    keys = ("q", "log_f", "i", "dO", "h0", "dhT")

    def step(t):
        sv = L.new_saved(t["q"])
        o, hT = L.fwd(t["q"], t["log_f"], t["i"], t["h0"], want_hT=True, chunk=64, saved=sv)
        dq, dlf, di, dh0 = L.bwd(t["q"], t["log_f"], t["i"], t["dO"], t["h0"], t["dhT"], want_dh0=True, chunk=64,
                                 saved=sv)
        return o, hT, dq, dlf, di, dh0

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # warm-up outside the capture (library load, kernel attributes)
        step(g)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = step(g)
    for k in keys:
        g[k].copy_(inp2[k].cuda())
    graph.replay()
    torch.cuda.synchronize()
    ref = step({k: inp2[k].cuda() for k in keys})
    torch.cuda.synchronize()
    assert L.device_status() == L.OK
    for a, b in zip(outs, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,T,H,d", [(8, 512, 16, 128), (2, 300, 3, 128), (2, 260, 2, 256)],
                         ids=["pair_per_cta", "segments", "wide_reduce_add"])
def test_three_runs_are_bitwise_identical(cuda, B, T, H, d):
    # determinism: the training pair run three times on the same inputs gives the same bits (no
    # order-dependent accumulation anywhere: the fix-ups add in a fixed order, and the 256-wide
    # shares are two addends per element)
    inp = I.make_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=81, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    g = to_cuda(inp)
    runs = []
    for _ in range(3):
        sv = L.new_saved(g["q"])
        o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, chunk=64, saved=sv)
        r = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, chunk=64, saved=sv)
        runs.append((o, hT) + tuple(r))
    torch.cuda.synchronize()
    assert L.device_status() == L.OK
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)
