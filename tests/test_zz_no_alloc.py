"""hgrn2_bwd_noalloc: the backward without a caller-supplied workspace.

This entry point serves callers that cannot hand the library a device buffer
(a plain C host program with no device allocator of its own, or a service that
must not allocate device memory once running, since cudaMalloc/cudaFree
synchronise the device).  Its scratch is a fixed array inside the library.
The test calls it through the C ABI and checks it against hgrn2_bwd on the
same inputs, twice in a row (the second call sees the first call's leftovers in
the shared scratch array, with different sizes and options), and against the
fp64 oracle, so that a fault shared by both library backwards cannot pass.  The
file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, tol

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _run_noalloc(lib, g, dtype, chunk, want_dh0):
    q, lf, x, dO = g["q"], g["log_f"], g["i"], g["dO"]
    B, T, H, dk = q.shape
    dv = x.shape[-1]
    dq, dlf, di = torch.empty_like(q), torch.empty_like(q), torch.empty_like(x)
    dh0 = torch.empty((B, H, dk, dv), device=q.device) if want_dh0 else None
    st = lib.hgrn2_bwd_noalloc(_p(q), _p(lf), _p(x), _p(g.get("h0")), _p(dO), _p(g.get("dhT")),
                               _p(dq), _p(dlf), _p(di), _p(dh0), B, T, H, dk, dv, chunk,
                               L.BF16 if dtype == torch.bfloat16 else L.FP32,
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.OK, L.status_string(st)
    return dq, dlf, di, dh0


@pytest.mark.parametrize("calls", [
    # two calls in a row: (dtype, B, T, H, d, lb, h0/dhT sigma, chunk)
    ((torch.bfloat16, 2, 300, 3, 128, 0.9, 0.1, 64), (torch.bfloat16, 1, 513, 5, 128, 0.5, 0.0, 128)),
    ((torch.float32, 1, 100, 2, 32, 0.0, 0.5, 32), (torch.bfloat16, 3, 129, 2, 128, 0.95, 0.2, 64)),
    # 64-wide heads: the no-alloc backward takes the exact route, hgrn2_bwd the tensor cores
    ((torch.bfloat16, 2, 300, 3, 64, 0.9, 0.1, 64), (torch.bfloat16, 1, 200, 4, 64, 0.5, 0.0, 128)),
])
def test_noalloc_matches_workspace_backward(cuda, calls):
    lib = L.load_library()
    for n, (dtype, B, T, H, d, lb, sig, chunk) in enumerate(calls):
        inp = I.make_inputs(B, T, H, d, d, dtype, lb, seed=500 + n + T, h0_sigma=sig, with_dO=True, dhT_sigma=sig)
        g = {k: v.cuda() for k, v in inp.items()}
        want_dh0 = sig > 0
        got = _run_noalloc(lib, g, dtype, chunk, want_dh0)
        ref = L.bwd(g["q"], g["log_f"], g["i"], g["dO"], g.get("h0"), g.get("dhT"), want_dh0=want_dh0, chunk=chunk)
        torch.cuda.synchronize()
        for name, a, r in zip(("dq", "dlog_f", "di", "dh0"), got, ref):
            if r is None:
                continue
            # the metric of the inputs' dtype for every output, as in the oracle parity tests: for
            # 64-wide bf16 heads the two calls take different routes (exact / tensor cores)
            e = err(np64(a), np64(r), dtype)
            assert e <= tol(dtype), (n, name, e)
        # and against the oracle, every (b, h) pair whole
        pairs = [(b, h) for b in range(B) for h in range(H)]
        orc = oracle_heads(inp, pairs, want_bwd=True, dhT=inp.get("dhT"))
        for k, (b, h) in enumerate(pairs):
            for name, a in zip(("dq", "dlog_f", "di", "dh0"), got):
                if a is None:
                    continue
                sl = a[b, h] if name == "dh0" else a[b, :, h]
                e = err(np64(sl), orc[name][k], dtype)
                assert e <= tol(dtype), ("oracle", n, name, b, h, e)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda):
    lib = L.load_library()
    vp = ctypes.c_void_p(16)
    # B*H = 4096 pairs at d_k = 128 need 2 MiB of scratch (> 1 MiB): refused before any launch
    st = lib.hgrn2_bwd_noalloc(vp, vp, vp, None, vp, None, vp, vp, vp, None, 64, 8, 64, 128, 128, 64, L.BF16,
                               None)
    assert st == L.ERR_UNSUPPORTED
