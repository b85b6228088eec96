"""Out-of-bounds writes, checked with guard canaries (compute-sanitizer is closed on this machine).

Every output tensor of a call is carved out of a larger buffer whose margins before and after
it are filled with a sentinel bit pattern; after the call the margins must hold exactly the
sentinel.  The calls are the ones whose kernels store with row masks or past ragged tails:
packed sequences (a sequence's last chunk is stored row by row), ragged T (TMA stores of the
last chunk), heads wider than 128 (column copies and partial sums), 64-wide heads (one 64-column
box per tile), the scalar-decay variant, the decode step and its backward, and the slice state
maps.  The margins are 4 KB: a store past the end of a row, a tile or a tensor lands in them.
"""
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I

pytestmark = pytest.mark.gpu

PAD = 4096   # bytes of sentinel before and after every output
SENTINEL = 0x5A


class Guarded:
    """Output tensors with sentinel margins on both sides."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        buf = torch.full((PAD + nbytes + PAD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[PAD:PAD + nbytes].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        for buf, nbytes in self.bufs:
            head, tail = buf[:PAD], buf[PAD + nbytes:]
            assert torch.all(head == SENTINEL), "write before an output"
            assert torch.all(tail == SENTINEL), "write after an output"


def _fwd_bwd(G, inp, chunk, saved):
    # every call through the C ABI, so that all outputs (the saved buffer included) sit inside
    # guarded buffers
    q, lf, x, dO = (inp[k] for k in ("q", "log_f", "i", "dO"))
    B, T, H, dk = q.shape
    dv = x.shape[-1]
    lib = L.load_library()
    p = lambda t: None if t is None else t.data_ptr()
    dt = L.BF16 if q.dtype == torch.bfloat16 else L.FP32
    stream = torch.cuda.current_stream().cuda_stream
    o = G.empty((B, T, H, dv), q.dtype)
    hT = G.empty((B, H, dk, dv), torch.float32)
    wsf = torch.empty(max(L.workspace_size(B, T, H, dk, dv, chunk, q.dtype, False), 16), dtype=torch.uint8,
                      device="cuda")
    if saved:
        n = L.saved_size(B, T, H, dk, dv, q.dtype)
        sv = G.empty((n,), torch.uint8)
        st = lib.hgrn2_fwd_train(p(q), p(lf), p(x), p(inp.get("h0")), p(o), p(hT), p(sv), n, B, T, H, dk, dv, chunk,
                                 dt, p(wsf), wsf.numel(), stream)
    else:
        st = lib.hgrn2_fwd(p(q), p(lf), p(x), p(inp.get("h0")), p(o), p(hT), B, T, H, dk, dv, chunk, dt, p(wsf),
                           wsf.numel(), stream)
    assert st == L.OK, L.status_string(st)
    dq, dlf = G.empty((B, T, H, dk), q.dtype), G.empty((B, T, H, dk), q.dtype)
    di, dh0 = G.empty((B, T, H, dv), q.dtype), G.empty((B, H, dk, dv), torch.float32)
    ws = torch.empty(max(L.workspace_size(B, T, H, dk, dv, chunk, q.dtype, 2 if saved else True), 16),
                     dtype=torch.uint8, device="cuda")
    if saved:
        st = lib.hgrn2_bwd_saved(p(q), p(lf), p(x), p(inp.get("h0")), p(sv), sv.numel(), p(dO), p(inp.get("dhT")),
                                 p(dq), p(dlf), p(di), p(dh0), B, T, H, dk, dv, chunk, dt, p(ws), ws.numel(), stream)
    else:
        st = lib.hgrn2_bwd(p(q), p(lf), p(x), p(inp.get("h0")), p(dO), p(inp.get("dhT")), p(dq), p(dlf), p(di),
                           p(dh0), B, T, H, dk, dv, chunk, dt, p(ws), ws.numel(), stream)
    assert st == L.OK, L.status_string(st)


@pytest.mark.parametrize("dtype,B,T,H,d,saved", [
    (torch.bfloat16, 1, 300, 3, 128, True),     # ragged T on the tensor cores
    (torch.bfloat16, 2, 129, 2, 128, False),    # one token past a chunk, recompute backward
    (torch.bfloat16, 1, 200, 2, 64, True),      # 64-wide heads
    (torch.bfloat16, 1, 130, 2, 256, True),     # 256-wide heads (as 128-wide blocks)
    (torch.float32, 2, 77, 2, 48, False),       # the exact route, ragged everything
])
def test_fwd_bwd_write_inside_their_outputs(cuda, dtype, B, T, H, d, saved):
    inp = I.make_inputs(B, T, H, d, d, dtype, 0.9, seed=1700 + T, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    G = Guarded()
    _fwd_bwd(G, {k: v.cuda() for k, v in inp.items()}, 64, saved)
    G.check()
    assert L.device_status() == L.OK


def test_packed_sequences_write_inside_their_outputs(cuda):
    lens = [5, 128, 129, 300, 1]
    inp = I.make_varlen(lens, 2, 128, 128, torch.bfloat16, 0.9, seed=1710, h0_sigma=0.1, with_dO=True, dhT_sigma=0.1)
    g = {k: v.cuda() for k, v in inp.items()}
    q, lf, x, dO, cu = g["q"], g["log_f"], g["i"], g["dO"], g["cu_seqlens"]
    G = Guarded()
    o = G.empty(tuple(x.shape), x.dtype)
    sv = L.new_saved_varlen(q, cu)
    L.fwd_varlen(q, lf, x, cu, g["h0"], want_hT=True, chunk=64, out=o, saved=sv)
    dq, dlf, di, dh0 = L.bwd_varlen(q, lf, x, dO, cu, g["h0"], g["dhT"], want_dh0=True, chunk=64, saved=sv)
    G.check()
    # the gradients were allocated by the binding: check them against a guarded copy of the call
    G2 = Guarded()
    outs = [G2.empty(tuple(t.shape), t.dtype) for t in (dq, dlf, di)]
    lib = L.load_library()
    p = lambda t: None if t is None else t.data_ptr()
    nseq, total = len(lens), q.shape[0]
    ws = torch.empty(max(L.workspace_size_varlen(nseq, total, 2, 128, 128, 64), 16), dtype=torch.uint8, device="cuda")
    st = lib.hgrn2_bwd_varlen(p(q), p(lf), p(x), p(g["h0"]), p(sv), sv.numel(), p(dO), p(g["dhT"]), p(outs[0]),
                              p(outs[1]), p(outs[2]), None, p(cu), nseq, total, 2, 128, 128, 64, L.BF16, p(ws),
                              ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == L.OK, L.status_string(st)
    G2.check()
    for a, b in zip(outs, (dq, dlf, di)):
        assert torch.equal(a, b)


def test_scalar_decay_step_and_state_maps_write_inside_their_outputs(cuda):
    G = Guarded()
    # scalar decay, ragged T, tensor cores
    s = {k: v.cuda() for k, v in I.make_scalar_inputs(1, 300, 2, 128, 128, torch.bfloat16, 0.9, seed=1720).items()}
    o = G.empty((1, 300, 2, 128), torch.bfloat16)
    hT = G.empty((1, 2, 128, 128), torch.float32)
    lib = L.load_library()
    p = lambda t: None if t is None else t.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.hgrn2_scalar_fwd(p(s["q"]), p(s["k"]), p(s["v"]), p(s["log_g"]), None, p(o), p(hT), 1, 300, 2, 128, 128,
                              L.BF16, stream)
    assert st == L.OK
    # decode step (dv = 12: a partial column group) and its backward
    d = I.make_decode(3, 2, 100, 12, 1, torch.bfloat16, 0.8, seed=1721)
    S = G.empty((3, 2, 100, 12), torch.float32)
    S.copy_(d["S"].cuda())
    o1 = G.empty((3, 2, 12), torch.bfloat16)
    qt, lft, xt = (d[k][0].cuda() for k in ("q", "log_f", "i"))
    assert lib.hgrn2_step(p(qt), p(lft), p(xt), p(S), p(o1), 3, 2, 100, 12, L.BF16, stream) == L.OK
    dq, dlf, di = (G.empty((3, 2, n), torch.bfloat16) for n in (100, 100, 12))
    dS = G.empty((3, 2, 100, 12), torch.float32)
    dO = torch.randn(3, 2, 12, device="cuda").to(torch.bfloat16)
    assert lib.hgrn2_step_bwd(p(qt), p(lft), p(xt), p(S), p(dO), None, p(dS), p(dq), p(dlf), p(di), 3, 2, 100, 12,
                              L.BF16, stream) == L.OK
    # slice state maps: tensor-core and CUDA-core routes, value columns not a multiple of 32
    for dk, dv in ((128, 128), (100, 40)):
        inp = {k: v.cuda() for k, v in I.make_inputs(1, 150, 2, dk, dv, torch.bfloat16, 0.5, seed=1722,
                                                      with_dO=True).items()}
        g_, U = G.empty((1, 2, dk), torch.float32), G.empty((1, 2, dk, dv), torch.float32)
        assert lib.hgrn2_state_map(p(inp["log_f"]), p(inp["i"]), 1, 150, 2, dk, dv, L.BF16, p(g_), p(U), stream) == L.OK
        assert lib.hgrn2_state_map_bwd(p(inp["q"]), p(inp["log_f"]), p(inp["dO"]), 1, 150, 2, dk, dv, L.BF16, p(g_),
                                       p(U), stream) == L.OK
    G.check()
    assert L.device_status() == L.OK
