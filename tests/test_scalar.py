"""GPU parity of the scalar-decay variant (hgrn2_scalar_fwd / hgrn2_scalar_bwd) against the
fp64 oracle: S_t = g_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t with one decay per head and token
("HGRN2: Gated Linear RNNs with State Expansion", §5 contrasts this per-head decay with its
per-dimension one).  Whole tensors at small sizes spanning several 32-token chunks and a
ragged tail; sampled (b, h) pairs at the training workload's size.
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, to_cuda
import oracle

pytestmark = pytest.mark.gpu

NAMES = ("o", "hT", "dq", "dk", "dv", "dlog_g", "dh0")


def _run(g, want_bwd=True):
    o, hT = L.scalar_fwd(g["q"], g["k"], g["v"], g["log_g"], g.get("h0"), want_hT=True)
    out = {"o": o, "hT": hT}
    if want_bwd:
        dq, dk, dv, dg, dh0 = L.scalar_bwd(g["q"], g["k"], g["v"], g["log_g"], g["dO"], g.get("h0"), g.get("dhT"),
                                           want_dh0=True)
        out.update(dq=dq, dk=dk, dv=dv, dlog_g=dg, dh0=dh0)
    assert L.device_status() == L.OK
    return out


def _ref(inp, b, h):
    sl = lambda t: None if t is None else np64(t[b:b + 1, :, h:h + 1])
    st = lambda t: None if t is None else np64(t[b:b + 1, h:h + 1])
    args = (sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_g"]))
    o, hT = oracle.sd_fwd(*args, st(inp.get("h0")))
    dq, dk, dv, dg, dh0 = oracle.sd_bwd(*args, sl(inp["dO"]), st(inp.get("h0")), st(inp.get("dhT")))
    return {"o": o[0, :, 0], "hT": hT[0, 0], "dq": dq[0, :, 0], "dk": dk[0, :, 0], "dv": dv[0, :, 0],
            "dlog_g": dg[0, :, 0], "dh0": dh0[0, 0]}


def _check(inp, got, pairs, dtype, bar):
    for b, h in pairs:
        ref = _ref(inp, b, h)
        for name in NAMES:
            t = got[name]
            g = np64(t[b, :, h] if t.dim() >= 3 and name not in ("hT", "dh0") else t[b, h])
            e = err(g, ref[name], dtype)
            assert e <= bar, (name, b, h, e)


CASES = [
    # dtype, B, T, H, dk, dv, lb, sigma
    (torch.float32, 1, 100, 2, 32, 16, 0.5, 0.5),
    (torch.float32, 2, 77, 1, 64, 48, 0.0, 0.5),
    (torch.float32, 1, 33, 2, 128, 128, 0.9, 0.0),
    (torch.float32, 1, 1, 3, 8, 4, 0.5, 0.5),
    (torch.bfloat16, 2, 300, 2, 128, 128, 0.95, 0.1),
    (torch.bfloat16, 1, 129, 3, 64, 64, 0.5, 0.0),
]


@pytest.mark.parametrize("case", CASES)
def test_scalar_matches_oracle(cuda, case):
    dtype, B, T, H, dk, dv, lb, sig = case
    inp = I.make_scalar_inputs(B, T, H, dk, dv, dtype, lb, seed=1100 + T + dk, h0_sigma=sig, with_dO=True,
                               dhT_sigma=sig)
    got = _run(to_cuda(inp))
    _check(inp, got, [(b, h) for b in range(B) for h in range(H)], dtype, 1e-4 if dtype == torch.float32 else 2e-2)


def test_scalar_strong_decay_is_exact(cuda):
    # log g = -12 per token: the cumulative decay inside a 32-token chunk reaches e^{-384}, far
    # past float range; the exponents the route forms are differences, all <= 0
    B, T, H, d = 1, 200, 2, 32
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.float32, 0.5, seed=1201, h0_sigma=0.5, with_dO=True,
                               dhT_sigma=0.5)
    inp["log_g"][:] = -12.0
    got = _run(to_cuda(inp))
    for name in NAMES:
        assert np.isfinite(np64(got[name])).all(), name
    for b, h in [(0, 0), (0, 1)]:
        ref = _ref(inp, b, h)
        for name in NAMES:
            g = np64(got[name][b, :, h] if name not in ("hT", "dh0") else got[name][b, h])
            if name == "dlog_g":
                # exact value g_t * O(1) ~ 1e-5, formed from O(1) summands q.dq - k.dk that cancel:
                # its error is bounded against the scale of those summands (the same degenerate
                # limit as d log f for f -> 0 on the per-dimension route)
                scale = np.max(np.abs((np64(inp["q"][b, :, h]) * ref["dq"]).sum(-1)))
                assert np.max(np.abs(g - ref[name])) <= 1e-4 * scale, name
            else:
                assert err(g, ref[name], torch.float32) <= 1e-4, name


def test_scalar_with_key_one_minus_gate_equals_hgrn2(cuda):
    # with every key dim equal to 1 - g_t and the gate shared by every dim, the scalar-decay call
    # and the HGRN2 call (tensor-core route) compute the same recurrence
    B, T, H, d = 2, 300, 2, 128
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=1202, h0_sigma=0.1)
    g = to_cuda(inp)
    lf = g["log_g"][..., None].expand(B, T, H, d).contiguous()
    k = (1.0 - torch.exp(g["log_g"].float()))[..., None].expand(B, T, H, d).to(torch.bfloat16).contiguous()
    o1, h1 = L.scalar_fwd(g["q"], k, g["v"], g["log_g"], g["h0"], want_hT=True)
    o2, h2 = L.fwd(g["q"], lf, g["v"], g["h0"], want_hT=True)
    # k rounded to bf16 on one side, formed in fp32 from log f on the other: compare at the bf16 bar
    assert err(np64(o1), np64(o2), torch.bfloat16) <= 2e-2
    assert err(np64(h1), np64(h2), torch.bfloat16) <= 2e-2


def test_scalar_training_workload_full_size_sampled(cuda):
    w = I.SCALAR_TRAIN
    inp = I.make_scalar_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.lb, seed=1203, with_dO=True)
    got = _run(to_cuda(inp))
    _check(inp, got, [(0, 0), (5, 9), (7, 15)], w.dtype, 2e-2)


def test_scalar_empty_sequence_passes_states_through(cuda):
    B, H, d = 2, 2, 16
    inp = I.make_scalar_inputs(B, 0, H, d, d, torch.float32, 0.5, seed=1204, h0_sigma=0.5, with_dO=True,
                               dhT_sigma=0.5)
    g = to_cuda(inp)
    got = _run(g)
    assert torch.equal(got["hT"], g["h0"]) and torch.equal(got["dh0"], g["dhT"])


@pytest.mark.parametrize("d,lb,strong", [(128, 0.5, None), (64, 0.9, None), (128, 0.0, None), (128, 0.5, "all"),
                                         (64, 0.9, "one")],
                         ids=["d128", "d64", "d128_lb0", "d128_strong_decay", "d64_one_flagged_head"])
def test_scalar_tensor_core_forward(cuda, d, lb, strong):
    # bf16 with d = 128 or 64 runs the scalar-decay instance of the tensor-core forward: chunk
    # passes and exact-route pairs are counted on the device.  A pair with a chunk whose summed
    # log g is below -150 (log g = -12 per token: e^{-1536} over a chunk) is recomputed by the
    # exact CUDA-core forward inside the same launch; the other pairs stay on the tensor cores.
    B, T, H = 2, 300, 3
    nt = (T + 127) // 128
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.bfloat16, lb, seed=1300 + d, h0_sigma=0.1)
    if strong == "all":
        inp["log_g"][:] = -12.0
    elif strong == "one":
        inp["log_g"][1, :, 0] = -12.0
    g = to_cuda(inp)
    L.counters(reset=True)
    o, hT = L.scalar_fwd(g["q"], g["k"], g["v"], g["log_g"], g["h0"], want_hT=True)
    c = L.counters(reset=True)
    exact = {None: 0, "all": B * H, "one": 1}[strong]
    assert c[0] == exact and c[1] == (B * H - exact) * nt and c[2] == 1, c
    assert L.device_status() == L.OK
    assert np.isfinite(np64(o)).all() and np.isfinite(np64(hT)).all()
    for b in range(B):
        for h in range(H):
            sl = lambda t: np64(t[b:b + 1, :, h:h + 1])
            ro, rh = oracle.sd_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_g"]),
                                   np64(inp["h0"][b:b + 1, h:h + 1]))
            assert err(np64(o[b, :, h]), ro[0, :, 0], torch.bfloat16) <= 2e-2, (b, h)
            assert err(np64(hT[b, h]), rh[0, 0], torch.bfloat16) <= 2e-2, (b, h)


@pytest.mark.parametrize("d", [128, 64])
def test_scalar_tensor_core_backward_with_a_flagged_head(cuda, d):
    # bf16 d = 128 / 64: the backward runs the forward again (chunk states saved into the workspace)
    # and the tensor-core reverse sweep: 4 launches (forward, reverse sweep, the exact route's two
    # kernels for flagged pairs).  Head (1, 2) has log g = -2 per token, a chunk total of -256,
    # past the factorised form's range (-150): it is recomputed on CUDA cores; the rest stays on
    # the tensor cores.  Every gradient must match the oracle.
    B, T, H = 2, 300, 3
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=1400 + d, h0_sigma=0.1, with_dO=True,
                               dhT_sigma=0.1)
    inp["log_g"][1, :, 2] = -2.0
    g = to_cuda(inp)
    L.counters(reset=True)
    dq, dk, dv, dg, dh0 = L.scalar_bwd(g["q"], g["k"], g["v"], g["log_g"], g["dO"], g["h0"], g["dhT"],
                                       want_dh0=True)
    c = L.counters(reset=True)
    assert c[2] == 4, c
    assert L.device_status() == L.OK
    o, hT = L.scalar_fwd(g["q"], g["k"], g["v"], g["log_g"], g["h0"], want_hT=True)
    got = {"o": o, "hT": hT, "dq": dq, "dk": dk, "dv": dv, "dlog_g": dg, "dh0": dh0}
    _check(inp, got, [(b, h) for b in range(B) for h in range(H)], torch.bfloat16, 2e-2)


@pytest.mark.parametrize("d", [128, 64])
def test_scalar_saved_state_pair(cuda, d):
    # the training pair: the forward keeps its chunk states, the backward reads them (one reverse
    # sweep plus the exact route's kernels for flagged pairs: 3 launches), with a flagged head
    B, T, H = 2, 300, 3
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=1500 + d, h0_sigma=0.1, with_dO=True,
                               dhT_sigma=0.1)
    inp["log_g"][0, :, 1] = -2.0
    g = to_cuda(inp)
    sv = L.new_scalar_saved(g["q"])
    assert sv is not None
    L.counters(reset=True)
    o, hT = L.scalar_fwd(g["q"], g["k"], g["v"], g["log_g"], g["h0"], want_hT=True, saved=sv)
    c_fwd = L.counters(reset=True)
    dq, dk, dv, dg, dh0 = L.scalar_bwd(g["q"], g["k"], g["v"], g["log_g"], g["dO"], g["h0"], g["dhT"], want_dh0=True,
                                       saved=sv)
    c_bwd = L.counters(reset=True)
    assert c_fwd[2] == 1 and c_bwd[2] == 3, (c_fwd, c_bwd)
    assert L.device_status() == L.OK
    got = {"o": o, "hT": hT, "dq": dq, "dk": dk, "dv": dv, "dlog_g": dg, "dh0": dh0}
    _check(inp, got, [(b, h) for b in range(B) for h in range(H)], torch.bfloat16, 2e-2)


def test_scalar_autograd_function(cuda):
    B, T, H, d = 1, 260, 2, 128
    inp = I.make_scalar_inputs(B, T, H, d, d, torch.bfloat16, 0.9, seed=1600, h0_sigma=0.1, with_dO=True,
                               dhT_sigma=0.1)
    g = to_cuda(inp)
    leaves = [g[n].clone().requires_grad_(True) for n in ("q", "k", "v", "log_g", "h0")]
    o, hT = L.scalar_decay(*leaves)
    loss = (o.float() * g["dO"].float()).sum() + (hT * g["dhT"]).sum()
    loss.backward()
    got = {"o": o.detach(), "hT": hT.detach(), "dq": leaves[0].grad, "dk": leaves[1].grad, "dv": leaves[2].grad,
           "dlog_g": leaves[3].grad, "dh0": leaves[4].grad}
    _check(inp, got, [(0, 0), (0, 1)], torch.bfloat16, 2e-2)
