"""GPU parity of packed variable-length sequences against the fp64 oracle.

Every sequence of a packed batch is an independent recurrence with its own
initial state ("HGRN2: Gated Linear RNNs with State Expansion", §2.1: the state
starts from h0 at the first token), so the oracle runs each sequence on its own
slice and the packed call must match it element by element.  Lengths cover the
edge cases of the 128-token chunking: empty, one token, one short of a chunk,
exactly a chunk, one past it, several chunks with a ragged tail.
"""
import numpy as np
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, to_cuda
import oracle

pytestmark = pytest.mark.gpu

EDGE_LENS = [300, 0, 1, 127, 128, 129, 45, 256]


def _oracle_seq(inp, s, h, want_bwd):
    """Oracle outputs of sequence s, head h: dict of float64 arrays."""
    cu = inp["cu_seqlens"].tolist()
    a, e = cu[s], cu[s + 1]
    sl = lambda t: None if t is None else np64(t[a:e, h:h + 1])[None]
    st = lambda t: None if t is None else np64(t[s:s + 1, h:h + 1])
    q, lf, x, h0 = sl(inp["q"]), sl(inp["log_f"]), sl(inp["i"]), st(inp.get("h0"))
    if e == a:   # an empty sequence passes its states through
        return {"o": None, "dq": None, "dlog_f": None, "di": None,
                "hT": h0[0, 0] if h0 is not None else 0.0,
                "dh0": st(inp["dhT"])[0, 0] if inp.get("dhT") is not None else 0.0}
    o, hT = oracle.fwd(q, lf, x, h0)
    r = {"o": o[0, :, 0], "hT": hT[0, 0]}
    if want_bwd:
        dq, dlf, di, dh0 = oracle.bwd(q, lf, x, sl(inp["dO"]), h0, st(inp.get("dhT")))
        r.update(dq=dq[0, :, 0], dlog_f=dlf[0, :, 0], di=di[0, :, 0], dh0=dh0[0, 0])
    return r


def _check(inp, got, seqs, heads, dtype, bar, want_bwd=True):
    cu = inp["cu_seqlens"].tolist()
    for s in seqs:
        a, e = cu[s], cu[s + 1]
        for h in heads:
            ref = _oracle_seq(inp, s, h, want_bwd)
            names = ("o", "hT", "dq", "dlog_f", "di", "dh0") if want_bwd else ("o", "hT")
            for name in names:
                t = got[name]
                if t is None or ref[name] is None:
                    continue
                g = np64(t[a:e, h] if name in ("o", "dq", "dlog_f", "di") else t[s, h])
                r = np.broadcast_to(np.asarray(ref[name], np.float64), g.shape)
                assert np.isfinite(g).all(), (name, s, h)
                if g.size == 0:
                    continue
                if not np.any(r):
                    assert np.max(np.abs(g)) == 0.0, (name, s, h)
                    continue
                e_ = err(g, r, dtype)
                assert e_ <= bar, (name, s, h, e - a, e_)


def _run(g, saved, chunk=64, want_bwd=True):
    sv = L.new_saved_varlen(g["q"], g["cu_seqlens"]) if saved else None
    o, hT = L.fwd_varlen(g["q"], g["log_f"], g["i"], g["cu_seqlens"], g.get("h0"), want_hT=True, chunk=chunk,
                         saved=sv)
    out = {"o": o, "hT": hT}
    if want_bwd:
        dq, dlf, di, dh0 = L.bwd_varlen(g["q"], g["log_f"], g["i"], g["dO"], g["cu_seqlens"], g.get("h0"),
                                        g.get("dhT"), want_dh0=True, chunk=chunk, saved=sv)
        out.update(dq=dq, dlog_f=dlf, di=di, dh0=dh0)
    assert L.device_status() == L.OK
    return out


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("states", [False, True], ids=["zero_state", "h0_dhT"])
def test_bf16_edge_lengths(cuda, saved, states):
    s = 0.1 if states else 0.0
    inp = I.make_varlen(EDGE_LENS, 2, 128, 128, torch.bfloat16, 0.9, seed=601, h0_sigma=s, with_dO=True,
                        dhT_sigma=s)
    got = _run(to_cuda(inp), saved)
    _check(inp, got, range(len(EDGE_LENS)), range(2), torch.bfloat16, 2e-2)


def test_bf16_launch_counts(cuda):
    # forward: the longest-first order of the sequences, then one tensor-core launch; the
    # backward reads that order and the chunk states from the saved buffer: one launch
    inp = I.make_varlen(EDGE_LENS, 2, 128, 128, torch.bfloat16, 0.9, seed=602, with_dO=True)
    g = to_cuda(inp)
    sv = L.new_saved_varlen(g["q"], g["cu_seqlens"])
    L.counters(reset=True)
    L.fwd_varlen(g["q"], g["log_f"], g["i"], g["cu_seqlens"], saved=sv)
    c_fwd = L.counters(reset=True)
    L.bwd_varlen(g["q"], g["log_f"], g["i"], g["dO"], g["cu_seqlens"], saved=sv)
    c_bwd = L.counters(reset=True)
    assert c_fwd[2] == 2 and c_bwd[2] == 1, (c_fwd, c_bwd)
    assert c_fwd[0] == 0 and c_bwd[0] == 0, (c_fwd, c_bwd)


@pytest.mark.parametrize("case", [(32, 16, 32), (64, 48, 16), (128, 128, 64)])
def test_fp32_exact_route(cuda, case):
    dk, dv, chunk = case
    lens = [100, 0, 33, 64, 1, 70]
    inp = I.make_varlen(lens, 2, dk, dv, torch.float32, 0.0, seed=603 + dk, h0_sigma=0.5, with_dO=True,
                        dhT_sigma=0.5)
    got = _run(to_cuda(inp), saved=False, chunk=chunk)
    _check(inp, got, range(len(lens)), range(2), torch.float32, 1e-4)


def test_bf16_strong_decay_sequence_takes_the_exact_route(cuda):
    # one sequence with gates shifted down (log-decay spans of ~-180 inside a chunk): its
    # (sequence, head) pairs are flagged and recomputed by the exact route inside the same
    # launches, from the sequence's own offset; the others stay on the tensor cores
    lens = [200, 300, 150]
    inp = I.make_varlen(lens, 2, 128, 128, torch.bfloat16, 0.9, seed=604, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    strong = I.make_inputs(1, 300, 2, 128, 128, torch.bfloat16, 0.0, seed=605, gate_shift=-1.0)
    inp["log_f"][200:500] = strong["log_f"][0]
    g = to_cuda(inp)
    L.counters(reset=True)
    got = _run(g, saved=True, chunk=128)
    c = L.counters(reset=True)
    assert c[0] == 2 * 2, c   # two heads of one sequence, once in each pass
    _check(inp, got, range(3), range(2), torch.bfloat16, 2e-2)


def test_bf16_many_sequences_more_pairs_than_sms(cuda):
    # documents of exponentially distributed length (mean 100) packed into 6000 tokens, 4 heads:
    # more (sequence, head) pairs than SMs
    lens = I.document_lengths(6000, 100, seed=606)
    assert len(lens) * 4 > 148 and sum(lens) == 6000
    inp = I.make_varlen(lens, 4, 128, 128, torch.bfloat16, 0.95, seed=607, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    got = _run(to_cuda(inp), saved=True)
    n = len(lens)
    rng = np.random.default_rng(3)
    seqs = sorted({0, n - 1, int(np.argmax(lens))} | set(rng.choice(n, 5, replace=False).tolist()))
    _check(inp, got, seqs, range(4), torch.bfloat16, 2e-2)


def test_all_sequences_empty(cuda):
    inp = I.make_varlen([0, 0, 0], 2, 128, 128, torch.bfloat16, 0.9, seed=608, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    got = _run(g, saved=True)
    assert torch.equal(got["hT"], g["h0"])
    assert torch.equal(got["dh0"], g["dhT"])


def test_packed_equal_lengths_match_the_batched_call(cuda):
    # B sequences of one length T packed back to back give, bit for bit, the batched call's
    # results when every chunk is full and B*H is large enough that the batched forward runs
    # one CTA per (b, h) (no sequence segments): the same kernels on the same tiles
    B, T, H = 8, 1024, 16
    inp = I.make_inputs(B, T, H, 128, 128, torch.bfloat16, 0.95, seed=609, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    sv = L.new_saved(g["q"])
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True, saved=sv)
    dq, dlf, di, dh0 = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g["h0"], g["dhT"], want_dh0=True, saved=sv)
    pk = lambda t: t.reshape(B * T, H, t.shape[-1])
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device="cuda")
    svp = L.new_saved_varlen(pk(g["q"]), cu)
    o2, hT2 = L.fwd_varlen(pk(g["q"]), pk(g["log_f"]), pk(g["i"]), cu, g["h0"], want_hT=True, saved=svp)
    r2 = L.bwd_varlen(pk(g["q"]), pk(g["log_f"]), pk(g["i"]), pk(g["dO"]), cu, g["h0"], g["dhT"], want_dh0=True,
                      saved=svp)
    assert L.device_status() == L.OK
    assert torch.equal(pk(o), o2) and torch.equal(hT, hT2)
    for a, b in zip((dq, dlf, di), r2[:3]):
        assert torch.equal(pk(a), b)
    assert torch.equal(dh0, r2[3])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_repacking_in_reverse_order_changes_no_bit(cuda, dtype):
    # each (sequence, head) pair depends on its own tokens and states only: packing the same
    # documents in the opposite order moves them to other token offsets, other chunk-state
    # slots and another launch order, and must reproduce every output bit for bit
    lens = EDGE_LENS
    inp = I.make_varlen(lens, 2, 128, 128, dtype, 0.9, seed=610, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    cu = inp["cu_seqlens"].tolist()
    order = list(reversed(range(len(lens))))
    rev = {k: torch.cat([inp[k][cu[s]:cu[s + 1]] for s in order]) for k in ("q", "log_f", "i", "dO")}
    rev["h0"], rev["dhT"] = inp["h0"][order].contiguous(), inp["dhT"][order].contiguous()
    rev["cu_seqlens"] = torch.tensor([0] + list(np.cumsum([lens[s] for s in order])), dtype=torch.int32)
    saved = dtype == torch.bfloat16
    a = _run(to_cuda(inp), saved=saved)
    b = _run(to_cuda(rev), saved=saved)
    rcu = rev["cu_seqlens"].tolist()
    for j, s in enumerate(order):
        for name in ("o", "dq", "dlog_f", "di"):
            assert torch.equal(a[name][cu[s]:cu[s + 1]], b[name][rcu[j]:rcu[j + 1]]), (name, s)
        for name in ("hT", "dh0"):
            assert torch.equal(a[name][s], b[name][j]), (name, s)


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_tokens_outside_every_sequence_are_left_untouched(cuda, saved):
    # cu_seqlens = [3, 3, 140, 140] over 200 tokens: sequence 1 is tokens 3..139, sequences 0
    # and 2 are empty; tokens 0..2 and 140..199 belong to none and keep what the buffers held
    H = 2
    inp = I.make_varlen([200], H, 128, 128, torch.bfloat16, 0.9, seed=611, h0_sigma=0.1, with_dO=True,
                        dhT_sigma=0.1)
    g = to_cuda(inp)
    nseq = 3
    cu = torch.tensor([3, 3, 140, 140], dtype=torch.int32, device="cuda")
    gen = torch.Generator().manual_seed(5)
    h0 = (0.1 * torch.randn((nseq, H, 128, 128), generator=gen)).cuda()
    dhT = (0.1 * torch.randn((nseq, H, 128, 128), generator=gen)).cuda()
    sentinel = 7.0
    o = torch.full((200, H, 128), sentinel, dtype=torch.bfloat16, device="cuda")
    sv = L.new_saved_varlen(g["q"], cu) if saved else None
    _, hT = L.fwd_varlen(g["q"], g["log_f"], g["i"], cu, h0, want_hT=True, out=o, saved=sv)
    dq, dlf, di, dh0 = L.bwd_varlen(g["q"], g["log_f"], g["i"], g["dO"], cu, h0, dhT, want_dh0=True, saved=sv)
    assert L.device_status() == L.OK
    outside = torch.cat([o[:3], o[140:]])
    assert torch.all(outside == sentinel)
    for s in (0, 2):   # empty: states pass through
        assert torch.equal(hT[s], h0[s]) and torch.equal(dh0[s], dhT[s])
    ref_in = {"q": inp["q"], "log_f": inp["log_f"], "i": inp["i"], "dO": inp["dO"],
              "h0": h0.cpu(), "dhT": dhT.cpu(), "cu_seqlens": torch.tensor([3, 3, 140, 140], dtype=torch.int32)}
    _check(ref_in, {"o": o, "hT": hT, "dq": dq, "dlog_f": dlf, "di": di, "dh0": dh0}, [1], range(H),
           torch.bfloat16, 2e-2)
