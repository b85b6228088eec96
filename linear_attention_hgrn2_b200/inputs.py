"""Seeded synthetic inputs for the HGRN2 recurrence.

This module is shared by the tests, the benchmark and the smoke check, and it
holds none of the recurrence's arithmetic: it only draws random tensors with
the shapes and value distributions of the workloads below and rounds them to
their storage dtype.  Both the CUDA path and the CPU oracle consume exactly the
tensors produced here (the oracle after an exact upcast to float64).

Forget gates follow the lower-bounded parameterisation of HGRN ("HGRN2: Gated
Linear RNNs with State Expansion", §2.2: each layer's forget gate is a learned
residual above a lower bound ``lb`` that rises with depth):

    f = lb + (1 - lb) * sigmoid(x),  x ~ N(0, 1),     log_f = log(f)

computed in float64, then rounded to the storage dtype.  q, i and dO are
N(0, 1); initial states are N(0, sigma^2) in float32.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: torch.dtype
    lb: float
    chunk: int
    h0_sigma: float = 0.0     # 0 => no initial state (zeros)
    want_hT: bool = False
    bwd: bool = False


# The five workloads, named by what they are.  Token tensors are [B, T, H, D].
TINY = Workload("tiny_fp32_B1_H2_T64_d16", 1, 2, 64, 16, 16, torch.float32, 0.0, 16)
FWD_LAYER = Workload("fwd_bf16_B4_H8_T2048_d128", 4, 8, 2048, 128, 128, torch.bfloat16, 0.5, 64)
TRAIN = Workload("train_fwdbwd_bf16_B8_H16_T2048_d128", 8, 16, 2048, 128, 128, torch.bfloat16,
                 0.95, 64, bwd=True)
LONG = Workload("long_fwd_bf16_B1_H8_T32768_d128", 1, 8, 32768, 128, 128, torch.bfloat16, 0.9, 64,
                h0_sigma=0.1, want_hT=True)
# decode: B=256 sequences, H=16, d=128, one token per step, 1000 steps, S ~ N(0,1)
DECODE = dict(name="decode_bf16_B256_H16_d128_1000steps", B=256, H=16, dk=128, dv=128,
              dtype=torch.bfloat16, lb=0.8, steps=1000, S_sigma=1.0)

# packed documents: the training step's 16,384 tokens per batch cut into documents of
# exponentially distributed length (mean 512 tokens), H=16, d=128, one state per document
VARLEN = dict(name="varlen_train_bf16_T16384_H16_d128_docmean512", total_T=16384, H=16, dk=128, dv=128,
              dtype=torch.bfloat16, lb=0.95, mean_len=512, chunk=64)

# the training workload with the first layer's forget-gate lower bound, lb = 0 (f = sigmoid(x))
TRAIN_LB0 = Workload("train_fwdbwd_bf16_B8_H16_T2048_d128_lb0", 8, 16, 2048, 128, 128, torch.bfloat16,
                     0.0, 64, bwd=True)

# the training workload's hidden size (2048) with 64-wide heads
TRAIN_D64 = Workload("train_fwdbwd_bf16_B8_H32_T2048_d64", 8, 32, 2048, 64, 64, torch.bfloat16, 0.95, 64, bwd=True)
# ... and with 256-wide heads
TRAIN_D256 = Workload("train_fwdbwd_bf16_B8_H8_T2048_d256", 8, 8, 2048, 256, 256, torch.bfloat16, 0.95, 64, bwd=True)
# ... and the long sequence's shape as a training pair (few (b,h): both directions in segments)
TRAIN_LONG = Workload("train_fwdbwd_bf16_B1_H8_T32768_d128", 1, 8, 32768, 128, 128, torch.bfloat16, 0.9, 64,
                      bwd=True)

WORKLOADS = {w.name: w for w in (TINY, FWD_LAYER, TRAIN, LONG, TRAIN_D64, TRAIN_D256)}


def _gen(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal(g: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x


def gate_log_f(x: np.ndarray, lb: float) -> np.ndarray:
    """log(lb + (1 - lb) * sigmoid(x)) in float64 (stable for lb = 0)."""
    x = x.astype(np.float64)
    if lb == 0.0:
        return -np.logaddexp(0.0, -x)          # log sigmoid(x)
    sig = 0.5 * (1.0 + np.tanh(0.5 * x))
    return np.log(lb + (1.0 - lb) * sig)


def _to(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: torch.dtype, lb: float,
                seed: int, h0_sigma: float = 0.0, with_dO: bool = False,
                dhT_sigma: float = 0.0, gate_shift: float = 0.0) -> dict:
    """CPU tensors q, log_f, i [B,T,H,*] in ``dtype``; optional h0, dO, dhT.

    The gate pre-activations are x ~ N(gate_shift, 1): a negative shift gives forget gates
    near 0 (decays far stronger than the workloads', for edge cases).
    Draw order (fixed): q, i, gate pre-activations, dO, h0, dhT."""
    g = _gen(seed)
    out = {}
    out["q"] = _to(_normal(g, (B, T, H, dk)), dtype)
    out["i"] = _to(_normal(g, (B, T, H, dv)), dtype)
    out["log_f"] = _to(gate_log_f(_normal(g, (B, T, H, dk)) + np.float32(gate_shift), lb), dtype)
    if with_dO:
        out["dO"] = _to(_normal(g, (B, T, H, dv)), dtype)
    if h0_sigma > 0:
        out["h0"] = torch.from_numpy(_normal(g, (B, H, dk, dv), h0_sigma))
    if dhT_sigma > 0:
        out["dhT"] = torch.from_numpy(_normal(g, (B, H, dk, dv), dhT_sigma))
    return out


def make_workload(w: Workload, seed: int) -> dict:
    return make_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.lb, seed,
                       h0_sigma=w.h0_sigma, with_dO=w.bwd)


def make_decode(B: int, H: int, dk: int, dv: int, steps: int, dtype: torch.dtype, lb: float,
                seed: int, S_sigma: float = 1.0, device: str = "cpu") -> dict:
    """Decode-step inputs: q, log_f [steps,B,H,dk], i [steps,B,H,dv] and S [B,H,dk,dv] fp32,
    plus g [steps,B,H,dk]: the gate pre-activations log_f was made from, rounded to dtype
    (for the lower-bounded-gate step, which takes them raw).

    On device='cpu' the draws use NumPy's PCG64 (bit-reproducible everywhere).
    On a CUDA device they use a seeded torch CUDA generator (for the large
    benchmark pool only; tests that compare with the oracle use the CPU draws)."""
    if device == "cpu":
        g = _gen(seed)
        q = _to(_normal(g, (steps, B, H, dk)), dtype)
        i = _to(_normal(g, (steps, B, H, dv)), dtype)
        x = _normal(g, (steps, B, H, dk))
        lf = _to(gate_log_f(x, lb), dtype)
        S = torch.from_numpy(_normal(g, (B, H, dk, dv), S_sigma))
        return {"q": q, "i": i, "log_f": lf, "S": S, "g": _to(x, dtype)}
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = torch.randn((steps, B, H, dk), generator=gen, device=device).to(dtype)
    i = torch.randn((steps, B, H, dv), generator=gen, device=device).to(dtype)
    x = torch.randn((steps, B, H, dk), generator=gen, device=device, dtype=torch.float64)
    lf = torch.log(lb + (1.0 - lb) * torch.sigmoid(x)).to(dtype)
    graw = x.to(dtype)
    del x
    S = torch.randn((B, H, dk, dv), generator=gen, device=device) * S_sigma
    return {"q": q, "i": i, "log_f": lf, "S": S, "g": graw}


def decode_state(B: int, H: int, dk: int, dv: int, seed: int, S_sigma: float = 1.0) -> torch.Tensor:
    """Initial decode state S [B,H,dk,dv] float32, N(0, S_sigma^2), for the streamed decode
    inputs below (its own PCG64 stream, so any number of steps can follow it)."""
    return torch.from_numpy(_normal(_gen(seed), (B, H, dk, dv), S_sigma))


def decode_token(B: int, H: int, dk: int, dv: int, dtype: torch.dtype, lb: float, seed: int, t: int) -> dict:
    """Inputs of decode step t alone: q, log_f [B,H,dk] and i [B,H,dv] in ``dtype``, drawn from
    a PCG64 stream keyed by (seed, t) in the order q, i, gate.  A long run of steps can then be
    generated one token at a time on the host, with no tensor holding every step."""
    g = np.random.Generator(np.random.PCG64([seed, t]))
    q = _to(_normal(g, (B, H, dk)), dtype)
    i = _to(_normal(g, (B, H, dv)), dtype)
    lf = _to(gate_log_f(_normal(g, (B, H, dk)), lb), dtype)
    return {"q": q, "i": i, "log_f": lf}


def make_varlen(lens, H: int, dk: int, dv: int, dtype: torch.dtype, lb: float, seed: int,
                h0_sigma: float = 0.0, with_dO: bool = False, dhT_sigma: float = 0.0) -> dict:
    """Packed variable-length sequences: CPU tensors q, log_f [total_T,H,dk], i (and dO)
    [total_T,H,dv] in ``dtype``, cu_seqlens int32 [nseq+1] (sequence s is tokens
    cu_seqlens[s] .. cu_seqlens[s+1]-1), optional h0, dhT [nseq,H,dk,dv] float32.

    The tokens are the draws of make_inputs(1, total_T, ...) with the same seed, so a
    sequence is a slice of one long stream; the states are drawn per sequence."""
    lens = [int(n) for n in lens]
    total = sum(lens)
    inp = make_inputs(1, total, H, dk, dv, dtype, lb, seed, with_dO=with_dO)
    out = {k: v[0] for k, v in inp.items()}
    out["cu_seqlens"] = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    g = _gen(seed + 1)
    if h0_sigma > 0:
        out["h0"] = torch.from_numpy(_normal(g, (len(lens), H, dk, dv), h0_sigma))
    if dhT_sigma > 0:
        out["dhT"] = torch.from_numpy(_normal(g, (len(lens), H, dk, dv), dhT_sigma))
    return out


def document_lengths(total: int, mean: int, seed: int, min_len: int = 1) -> list:
    """Lengths of documents packed into ``total`` tokens: exponential with the given mean
    (many short documents, a few long ones), at least ``min_len``; the last one is cut to
    fill ``total`` exactly."""
    g = _gen(seed)
    lens, used = [], 0
    while used < total:
        n = max(min_len, int(g.exponential(mean)))
        n = min(n, total - used)
        lens.append(n)
        used += n
    return lens


def make_step_grads(B: int, H: int, dk: int, dv: int, dtype: torch.dtype, seed: int,
                    dS_sigma: float = 1.0) -> dict:
    """Upstream gradients of one decode step: dO [B,H,dv] in ``dtype`` (N(0,1)) and
    dS [B,H,dk,dv] float32 (N(0, dS_sigma^2)), drawn in that order."""
    g = _gen(seed)
    return {"dO": _to(_normal(g, (B, H, dv)), dtype),
            "dS": torch.from_numpy(_normal(g, (B, H, dk, dv), dS_sigma))}


# Scalar-decay variant at the training workload's shape: one decay per head and token,
# g = lb + (1 - lb) sigmoid(x) as for the per-dimension gates, an explicit key k ~ N(0, 1/d_k)
SCALAR_TRAIN = Workload("scalar_fwdbwd_bf16_B8_H16_T2048_d128", 8, 16, 2048, 128, 128, torch.bfloat16, 0.95,
                        32, bwd=True)


def make_scalar_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: torch.dtype, lb: float, seed: int,
                       h0_sigma: float = 0.0, with_dO: bool = False, dhT_sigma: float = 0.0) -> dict:
    """CPU tensors for the scalar-decay variant: q, k [B,T,H,dk], v [B,T,H,dv], log_g [B,T,H]
    in ``dtype``; optional h0, dO, dhT.  Draw order (fixed): q, k, v, gate, dO, h0, dhT."""
    g = _gen(seed)
    out = {"q": _to(_normal(g, (B, T, H, dk)), dtype),
           "k": _to(_normal(g, (B, T, H, dk), 1.0 / np.sqrt(dk)), dtype),
           "v": _to(_normal(g, (B, T, H, dv)), dtype)}
    out["log_g"] = _to(gate_log_f(_normal(g, (B, T, H)), lb), dtype)
    if with_dO:
        out["dO"] = _to(_normal(g, (B, T, H, dv)), dtype)
    if h0_sigma > 0:
        out["h0"] = torch.from_numpy(_normal(g, (B, H, dk, dv), h0_sigma))
    if dhT_sigma > 0:
        out["dhT"] = torch.from_numpy(_normal(g, (B, H, dk, dv), dhT_sigma))
    return out
