"""Error metrics and oracle helpers shared by the GPU parity tests.

Tolerances (the accuracy bar set for this method: fp32 relative, bf16 normalised max-abs):
  * float32 inputs: max relative error <= 1e-4, measured element-wise as
        max_i |g_i - r_i| / max(|r_i|, FP32_FLOOR * max_j |r_j|)
    The floor keeps elements that are ~0 from dividing by ~0: an element-wise
    ratio is unbounded there for any finite-precision arithmetic.  Elements
    below FP32_FLOOR of the tensor's largest magnitude are thus held to an
    absolute error of 1e-4 * FP32_FLOOR * max|r|.  test_fp32_metric.py measures
    a plain token-by-token float32 recurrence under each candidate floor (1.9e-4
    with a 1e-3*rms floor, about 7e-5 with 1e-3*max, about 7e-6 with 1e-2*max);
  * bfloat16 inputs with a float32 state: normalised max-abs error <= 2e-2,
        max_i |g_i - r_i| / max_i |r_i|,
    per output tensor.
The oracle consumes exactly the (already rounded) inputs the GPU sees, upcast
to float64, so input rounding is never counted as error.
"""
import numpy as np
import torch

import oracle

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2
FP32_FLOOR = 1e-2   # relative to max|r|


def np64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def rel_err(g, r, floor=None):
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    if r.size == 0:
        return 0.0
    fl = FP32_FLOOR if floor is None else floor
    den = np.maximum(np.abs(r), fl * np.max(np.abs(r)) + 1e-300)
    return float(np.max(np.abs(g - r) / den))


def norm_max_abs(g, r):
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    if r.size == 0:
        return 0.0
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


def err(g, r, dtype):
    return rel_err(g, r) if dtype == torch.float32 else norm_max_abs(g, r)


def tol(dtype):
    return TOL_FP32 if dtype == torch.float32 else TOL_BF16


def oracle_heads(inp, pairs, want_bwd=False, dhT=None):
    """Runs the oracle on the selected (b, h) pairs only (each pair is independent).

    Returns dict name -> list of per-pair arrays ([T, D] for token tensors, [dk, dv] for states)."""
    res = {k: [] for k in ("o", "hT", "dq", "dlog_f", "di", "dh0")}
    for b, h in pairs:
        sl = lambda t: None if t is None else np64(t[b:b + 1, :, h:h + 1])
        st = lambda t: None if t is None else np64(t[b:b + 1, h:h + 1])
        q, lf, x = sl(inp["q"]), sl(inp["log_f"]), sl(inp["i"])
        h0 = st(inp.get("h0"))
        o, hT = oracle.fwd(q, lf, x, h0)
        res["o"].append(o[0, :, 0])
        res["hT"].append(hT[0, 0])
        if want_bwd:
            dq, dlf, di, dh0 = oracle.bwd(q, lf, x, sl(inp["dO"]), h0, st(dhT))
            res["dq"].append(dq[0, :, 0])
            res["dlog_f"].append(dlf[0, :, 0])
            res["di"].append(di[0, :, 0])
            res["dh0"].append(dh0[0, 0])
    return res


def to_cuda(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
