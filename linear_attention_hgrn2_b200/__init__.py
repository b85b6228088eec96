"""Python binding of libhgrn2.so, the B200 (sm_100a) HGRN2 recurrence library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/hgrn2.h``.  PyTorch supplies
device memory and the current CUDA stream.  There is no CPU fallback: if the
shared library is missing or cannot be loaded, every call raises.

Per batch b and head h, with f = exp(log_f) and k = 1 - f ("HGRN2: Gated
Linear RNNs with State Expansion", §2.1, §3.2):

    S_t = Diag(f_t) S_{t-1} + k_t i_t^T,      o_t = S_t^T q_t

Token tensors are [B, T, H, D]; states [B, H, d_k, d_v] float32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhgrn2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(6)
FP32, BF16 = 0, 1

# Every extern "C" symbol of include/hgrn2.h.
EXPORTS = ("hgrn2_workspace_size", "hgrn2_fwd", "hgrn2_bwd", "hgrn2_saved_size", "hgrn2_fwd_train",
           "hgrn2_bwd_saved", "hgrn2_bwd_noalloc", "hgrn2_workspace_size_varlen", "hgrn2_saved_size_varlen",
           "hgrn2_fwd_varlen", "hgrn2_bwd_varlen", "hgrn2_step", "hgrn2_step_lb", "hgrn2_step_bwd",
           "hgrn2_step_lb_bwd", "hgrn2_get_device_status", "hgrn2_get_counters", "hgrn2_status_string",
           "hgrn2_version", "hgrn2_selftest_wait_timeout", "hgrn2_scalar_workspace_size", "hgrn2_scalar_fwd",
           "hgrn2_scalar_bwd", "hgrn2_scalar_saved_size", "hgrn2_scalar_fwd_train", "hgrn2_scalar_bwd_saved",
           "hgrn2_state_map", "hgrn2_state_map_bwd", "hgrn2_affine_scan")

_lib = None


class HGRN2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libhgrn2.so (raises if it is absent: build it with
    ``python -m linear_attention_hgrn2_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libhgrn2.so not found at {path}; run `python -m linear_attention_hgrn2_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.hgrn2_workspace_size.argtypes = [i32] * 7 + [i32]
    lib.hgrn2_workspace_size.restype = sz
    lib.hgrn2_fwd.argtypes = [vp] * 6 + [i32] * 7 + [vp, sz, vp]
    lib.hgrn2_fwd.restype = i32
    lib.hgrn2_bwd.argtypes = [vp] * 10 + [i32] * 7 + [vp, sz, vp]
    lib.hgrn2_bwd.restype = i32
    lib.hgrn2_saved_size.argtypes = [i32] * 6
    lib.hgrn2_saved_size.restype = sz
    lib.hgrn2_fwd_train.argtypes = [vp] * 7 + [sz] + [i32] * 7 + [vp, sz, vp]
    lib.hgrn2_fwd_train.restype = i32
    lib.hgrn2_bwd_saved.argtypes = [vp] * 5 + [sz] + [vp] * 6 + [i32] * 7 + [vp, sz, vp]
    lib.hgrn2_bwd_saved.restype = i32
    lib.hgrn2_bwd_noalloc.argtypes = [vp] * 10 + [i32] * 7 + [vp]
    lib.hgrn2_bwd_noalloc.restype = i32
    lib.hgrn2_workspace_size_varlen.argtypes = [i32] * 7
    lib.hgrn2_workspace_size_varlen.restype = sz
    lib.hgrn2_saved_size_varlen.argtypes = [i32] * 6
    lib.hgrn2_saved_size_varlen.restype = sz
    lib.hgrn2_fwd_varlen.argtypes = [vp] * 7 + [i32] * 7 + [vp, sz, vp, sz, vp]
    lib.hgrn2_fwd_varlen.restype = i32
    lib.hgrn2_bwd_varlen.argtypes = [vp] * 5 + [sz] + [vp] * 7 + [i32] * 7 + [vp, sz, vp]
    lib.hgrn2_bwd_varlen.restype = i32
    lib.hgrn2_step.argtypes = [vp] * 5 + [i32] * 5 + [vp]
    lib.hgrn2_step_bwd.argtypes = [vp] * 10 + [i32] * 5 + [vp]
    lib.hgrn2_step_bwd.restype = i32
    lib.hgrn2_step_lb_bwd.argtypes = [vp] * 3 + [ctypes.c_float] + [vp] * 7 + [i32] * 5 + [vp]
    lib.hgrn2_step_lb_bwd.restype = i32
    lib.hgrn2_step.restype = i32
    lib.hgrn2_step_lb.argtypes = [vp] * 3 + [ctypes.c_float] + [vp] * 2 + [i32] * 5 + [vp]
    lib.hgrn2_step_lb.restype = i32
    lib.hgrn2_get_device_status.argtypes = [vp]
    lib.hgrn2_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    lib.hgrn2_scalar_workspace_size.argtypes = [i32] * 7
    lib.hgrn2_scalar_saved_size.argtypes = [i32] * 6
    lib.hgrn2_scalar_saved_size.restype = sz
    lib.hgrn2_scalar_fwd_train.argtypes = [vp] * 8 + [sz] + [i32] * 6 + [vp]
    lib.hgrn2_scalar_fwd_train.restype = i32
    lib.hgrn2_scalar_bwd_saved.argtypes = [vp] * 6 + [sz] + [vp] * 7 + [i32] * 6 + [vp, sz, vp]
    lib.hgrn2_scalar_bwd_saved.restype = i32
    lib.hgrn2_scalar_workspace_size.restype = sz
    lib.hgrn2_scalar_fwd.argtypes = [vp] * 7 + [i32] * 6 + [vp]
    lib.hgrn2_scalar_fwd.restype = i32
    lib.hgrn2_scalar_bwd.argtypes = [vp] * 12 + [i32] * 6 + [vp, sz, vp]
    lib.hgrn2_scalar_bwd.restype = i32
    lib.hgrn2_selftest_wait_timeout.restype = i32
    lib.hgrn2_state_map.argtypes = [vp] * 2 + [i32] * 6 + [vp] * 3
    lib.hgrn2_state_map.restype = i32
    lib.hgrn2_state_map_bwd.argtypes = [vp] * 3 + [i32] * 6 + [vp] * 3
    lib.hgrn2_state_map_bwd.restype = i32
    lib.hgrn2_affine_scan.argtypes = [vp] * 2 + [i32] * 4 + [vp] * 2 + [i32] * 4 + [vp]
    lib.hgrn2_affine_scan.restype = i32
    lib.hgrn2_get_device_status.restype = i32
    lib.hgrn2_get_counters.argtypes = [ctypes.POINTER(ctypes.c_longlong), i32, i32, vp]
    lib.hgrn2_get_counters.restype = i32
    lib.hgrn2_status_string.argtypes = [i32]
    lib.hgrn2_status_string.restype = ctypes.c_char_p
    lib.hgrn2_version.argtypes = []
    lib.hgrn2_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().hgrn2_status_string(status).decode()


def version() -> str:
    return load_library().hgrn2_version().decode()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _raise(status: int, where: str):
    if status != OK:
        raise HGRN2Error(status, where)


def workspace_size(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16, want_bwd=False) -> int:
    """want_bwd: False (forward), True (backward), or 2 (backward given saved states)."""
    n = load_library().hgrn2_workspace_size(B, T, H, dk, dv, chunk,
                                            BF16 if dtype == torch.bfloat16 else FP32, int(want_bwd))
    if n == ctypes.c_size_t(-1).value:
        raise HGRN2Error(ERR_INVALID_ARG, "hgrn2_workspace_size")
    return int(n)


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _caller_workspace(t: torch.Tensor) -> torch.Tensor:
    _check(t, "workspace", torch.uint8)
    return t


def saved_size(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Bytes of the buffer that fwd(..., saved=) fills for bwd(..., saved=); 0 when
    this configuration has no saved-state path (the backward then recomputes)."""
    n = load_library().hgrn2_saved_size(B, T, H, dk, dv, BF16 if dtype == torch.bfloat16 else FP32)
    if n == ctypes.c_size_t(-1).value:
        raise HGRN2Error(ERR_INVALID_ARG, "hgrn2_saved_size")
    return int(n)


def new_saved(q: torch.Tensor, dv: int | None = None) -> torch.Tensor | None:
    """An uninitialised saved-state buffer for a forward on q (None if not needed)."""
    B, T, H, dk = q.shape
    n = saved_size(B, T, H, dk, dk if dv is None else dv, q.dtype)
    return torch.empty(n, dtype=torch.uint8, device=q.device) if n else None


def fwd(q, log_f, i, h0=None, want_hT=False, chunk=64, out=None, workspace=None, saved=None):
    """o = HGRN2(q, log_f, i; h0) and optionally the final state hT.

    q, log_f: [B,T,H,dk]; i: [B,T,H,dv] (float32 or bfloat16, all the same);
    h0: [B,H,dk,dv] float32 or None.  saved: a uint8 CUDA buffer of saved_size()
    bytes (see new_saved) that receives the chunk states for bwd(..., saved=), or
    None.  Returns (o, hT or None)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = i.shape[-1]
    _check(q, "q")
    _check(log_f, "log_f", q.dtype, q.shape)
    _check(i, "i", q.dtype, (B, T, H, dv))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    o = out if out is not None else torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _check(o, "o", q.dtype, (B, T, H, dv))
    hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_hT else None
    nws = workspace_size(B, T, H, dk, dv, chunk, q.dtype, False)
    ws = _caller_workspace(workspace) if workspace is not None else _workspace(nws, q.device)
    if workspace is not None:
        nws = workspace.numel()   # the library checks it against what it needs
    if saved is not None:
        _check(saved, "saved", torch.uint8)
        st = lib.hgrn2_fwd_train(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(o), _ptr(hT), _ptr(saved),
                                 saved.numel(), B, T, H, dk, dv, chunk, _dt(q), _ptr(ws), nws, _stream())
        _raise(st, "hgrn2_fwd_train")
        return o, hT
    st = lib.hgrn2_fwd(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(o), _ptr(hT),
                       B, T, H, dk, dv, chunk, _dt(q), _ptr(ws), nws, _stream())
    _raise(st, "hgrn2_fwd")
    return o, hT


def bwd(q, log_f, i, dO, h0=None, dhT=None, want_dh0=False, chunk=64, workspace=None, saved=None):
    """Gradients (dq, dlog_f, di, dh0 or None) of L(o, hT) given dO (and dhT).

    saved: the buffer a fwd(..., saved=) on the same q, log_f, i, h0 filled (the
    states are then read instead of recomputed), or None."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = i.shape[-1]
    _check(q, "q")
    _check(log_f, "log_f", q.dtype, q.shape)
    _check(i, "i", q.dtype, (B, T, H, dv))
    _check(dO, "dO", q.dtype, (B, T, H, dv))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    if dhT is not None:
        _check(dhT, "dhT", torch.float32, (B, H, dk, dv))
    dq = torch.empty_like(q)
    dlf = torch.empty_like(q)
    di = torch.empty_like(i)
    dh0 = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_dh0 else None
    nws = workspace_size(B, T, H, dk, dv, chunk, q.dtype, 2 if saved is not None else True)
    ws = _caller_workspace(workspace) if workspace is not None else _workspace(nws, q.device)
    if workspace is not None:
        nws = workspace.numel()   # the library checks it against what it needs
    if saved is not None:
        _check(saved, "saved", torch.uint8)
        st = lib.hgrn2_bwd_saved(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(saved), saved.numel(),
                                 _ptr(dO), _ptr(dhT), _ptr(dq), _ptr(dlf), _ptr(di), _ptr(dh0),
                                 B, T, H, dk, dv, chunk, _dt(q), _ptr(ws), nws, _stream())
        _raise(st, "hgrn2_bwd_saved")
        return dq, dlf, di, dh0
    st = lib.hgrn2_bwd(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(dO), _ptr(dhT),
                       _ptr(dq), _ptr(dlf), _ptr(di), _ptr(dh0),
                       B, T, H, dk, dv, chunk, _dt(q), _ptr(ws), nws, _stream())
    _raise(st, "hgrn2_bwd")
    return dq, dlf, di, dh0


def _size_or_raise(n: int, where: str) -> int:
    if n == ctypes.c_size_t(-1).value:
        raise HGRN2Error(ERR_INVALID_ARG, where)
    return int(n)


def saved_size_varlen(nseq, total_T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Bytes of the saved-state buffer of fwd_varlen (0: no saved-state path)."""
    return _size_or_raise(load_library().hgrn2_saved_size_varlen(nseq, total_T, H, dk, dv,
                                                                  BF16 if dtype == torch.bfloat16 else FP32),
                          "hgrn2_saved_size_varlen")


def workspace_size_varlen(nseq, total_T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    return _size_or_raise(load_library().hgrn2_workspace_size_varlen(nseq, total_T, H, dk, dv, chunk,
                                                                      BF16 if dtype == torch.bfloat16 else FP32),
                          "hgrn2_workspace_size_varlen")


def new_saved_varlen(q: torch.Tensor, cu_seqlens: torch.Tensor, dv: int | None = None) -> torch.Tensor | None:
    """An uninitialised saved-state buffer for fwd_varlen on packed q [total_T,H,dk]."""
    total_T, H, dk = q.shape
    n = saved_size_varlen(cu_seqlens.numel() - 1, total_T, H, dk, dk if dv is None else dv, q.dtype)
    return torch.empty(n, dtype=torch.uint8, device=q.device) if n else None


def _check_varlen(q, log_f, i, cu_seqlens):
    _check(q, "q")
    if q.dim() != 3:
        raise ValueError("packed token tensors are [total_T, H, D]")
    total_T, H, dk = q.shape
    dv = i.shape[-1]
    _check(log_f, "log_f", q.dtype, q.shape)
    _check(i, "i", q.dtype, (total_T, H, dv))
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be [nseq + 1] with nseq >= 1")
    return total_T, H, dk, dv, cu_seqlens.numel() - 1


def fwd_varlen(q, log_f, i, cu_seqlens, h0=None, want_hT=False, chunk=64, out=None, saved=None):
    """Packed variable-length sequences: q, log_f [total_T,H,dk], i [total_T,H,dv];
    sequence s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 (int32 CUDA tensor), each
    with its own state (h0, hT: [nseq,H,dk,dv] float32).  saved: new_saved_varlen()
    or None.  Returns (o [total_T,H,dv], hT or None)."""
    lib = load_library()
    total_T, H, dk, dv, nseq = _check_varlen(q, log_f, i, cu_seqlens)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (nseq, H, dk, dv))
    o = out if out is not None else torch.empty((total_T, H, dv), dtype=q.dtype, device=q.device)
    _check(o, "o", q.dtype, (total_T, H, dv))
    hT = torch.empty((nseq, H, dk, dv), dtype=torch.float32, device=q.device) if want_hT else None
    nws = workspace_size_varlen(nseq, total_T, H, dk, dv, chunk, q.dtype)
    ws = _workspace(nws, q.device)
    if saved is not None:
        _check(saved, "saved", torch.uint8)
    st = lib.hgrn2_fwd_varlen(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(o), _ptr(hT), _ptr(cu_seqlens),
                              nseq, total_T, H, dk, dv, chunk, _dt(q), _ptr(saved),
                              0 if saved is None else saved.numel(), _ptr(ws), nws, _stream())
    _raise(st, "hgrn2_fwd_varlen")
    return o, hT


def bwd_varlen(q, log_f, i, dO, cu_seqlens, h0=None, dhT=None, want_dh0=False, chunk=64, saved=None):
    """Gradients (dq, dlog_f, di, dh0 or None) of packed sequences (see fwd_varlen)."""
    lib = load_library()
    total_T, H, dk, dv, nseq = _check_varlen(q, log_f, i, cu_seqlens)
    _check(dO, "dO", q.dtype, (total_T, H, dv))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (nseq, H, dk, dv))
    if dhT is not None:
        _check(dhT, "dhT", torch.float32, (nseq, H, dk, dv))
    dq = torch.empty_like(q)
    dlf = torch.empty_like(q)
    di = torch.empty_like(i)
    dh0 = torch.empty((nseq, H, dk, dv), dtype=torch.float32, device=q.device) if want_dh0 else None
    nws = workspace_size_varlen(nseq, total_T, H, dk, dv, chunk, q.dtype)
    ws = _workspace(nws, q.device)
    if saved is not None:
        _check(saved, "saved", torch.uint8)
    st = lib.hgrn2_bwd_varlen(_ptr(q), _ptr(log_f), _ptr(i), _ptr(h0), _ptr(saved),
                              0 if saved is None else saved.numel(), _ptr(dO), _ptr(dhT),
                              _ptr(dq), _ptr(dlf), _ptr(di), _ptr(dh0), _ptr(cu_seqlens),
                              nseq, total_T, H, dk, dv, chunk, _dt(q), _ptr(ws), nws, _stream())
    _raise(st, "hgrn2_bwd_varlen")
    return dq, dlf, di, dh0


def step(q, log_f, i, S, out=None):
    """One decode step: S <- Diag(f) S + k i^T in place; returns o = S^T q.

    q, log_f: [B,H,dk]; i: [B,H,dv]; S: [B,H,dk,dv] float32 (updated in place)."""
    lib = load_library()
    B, H, dk = q.shape
    dv = i.shape[-1]
    _check(q, "q")
    _check(log_f, "log_f", q.dtype, q.shape)
    _check(i, "i", q.dtype, (B, H, dv))
    _check(S, "S", torch.float32, (B, H, dk, dv))
    o = out if out is not None else torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = lib.hgrn2_step(_ptr(q), _ptr(log_f), _ptr(i), _ptr(S), _ptr(o), B, H, dk, dv, _dt(q), _stream())
    _raise(st, "hgrn2_step")
    return o


def step_lb(q, g, i, lb: float, S, out=None):
    """One decode step with the lower-bounded forget gate f = lb + (1 - lb) sigmoid(g)
    formed in the kernel from the raw gate logits g [B,H,dk]; otherwise as step()."""
    lib = load_library()
    B, H, dk = q.shape
    dv = i.shape[-1]
    _check(q, "q")
    _check(g, "g", q.dtype, q.shape)
    _check(i, "i", q.dtype, (B, H, dv))
    _check(S, "S", torch.float32, (B, H, dk, dv))
    o = out if out is not None else torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = lib.hgrn2_step_lb(_ptr(q), _ptr(g), _ptr(i), ctypes.c_float(lb), _ptr(S), _ptr(o), B, H, dk, dv, _dt(q),
                           _stream())
    _raise(st, "hgrn2_step_lb")
    return o


def _step_bwd(fn, name, q, gate, i, S, dO, dS, lb, dS_out):
    lib = load_library()
    B, H, dk = q.shape
    dv = i.shape[-1]
    _check(q, "q")
    _check(gate, "gate", q.dtype, q.shape)
    _check(i, "i", q.dtype, (B, H, dv))
    _check(S, "S", torch.float32, (B, H, dk, dv))
    _check(dO, "dO", q.dtype, (B, H, dv))
    if dS is not None:
        _check(dS, "dS", torch.float32, (B, H, dk, dv))
    if dS_out is None:
        dS_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check(dS_out, "dS_prev", torch.float32, (B, H, dk, dv))
    dq = torch.empty_like(q)
    dg = torch.empty_like(q)
    di = torch.empty_like(i)
    args = [_ptr(q), _ptr(gate), _ptr(i)] + ([ctypes.c_float(lb)] if lb is not None else [])
    st = fn(*args, _ptr(S), _ptr(dO), _ptr(dS), _ptr(dS_out), _ptr(dq), _ptr(dg), _ptr(di), B, H, dk, dv, _dt(q),
            _stream())
    _raise(st, name)
    return dq, dg, di, dS_out


def step_bwd(q, log_f, i, S, dO, dS=None, dS_out=None):
    """Backward of step(): S is the state before the step, dO = dL/do, dS = dL/dS_new (None:
    zero).  Returns (dq, dlog_f, di, dS_prev); dS_out (may be dS, for in place) receives dS_prev."""
    return _step_bwd(load_library().hgrn2_step_bwd, "hgrn2_step_bwd", q, log_f, i, S, dO, dS, None, dS_out)


def step_lb_bwd(q, g, i, lb: float, S, dO, dS=None, dS_out=None):
    """Backward of step_lb(): as step_bwd, returning dL/dg in place of dlog_f."""
    return _step_bwd(load_library().hgrn2_step_lb_bwd, "hgrn2_step_lb_bwd", q, g, i, S, dO, dS, lb, dS_out)


def scalar_saved_size(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Bytes of the buffer scalar_fwd(..., saved=) fills for scalar_bwd(..., saved=) (0: none)."""
    return _size_or_raise(load_library().hgrn2_scalar_saved_size(B, T, H, dk, dv,
                                                                  BF16 if dtype == torch.bfloat16 else FP32),
                          "hgrn2_scalar_saved_size")


def new_scalar_saved(q: torch.Tensor, dv: int | None = None) -> torch.Tensor | None:
    """An uninitialised saved-state buffer for a scalar-decay forward on q (None if not needed)."""
    B, T, H, dk = q.shape
    n = scalar_saved_size(B, T, H, dk, dk if dv is None else dv, q.dtype)
    return torch.empty(n, dtype=torch.uint8, device=q.device) if n else None


def scalar_fwd(q, k, v, log_g, h0=None, want_hT=False, saved=None):
    """Scalar-decay variant: S_t = g_t S_{t-1} + k_t v_t^T, o_t = S_t^T q_t, g_t = exp(log_g_t).

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; log_g: [B,T,H] (same dtype); h0: [B,H,dk,dv] float32 or
    None.  saved: new_scalar_saved() buffer that receives the chunk states for
    scalar_bwd(..., saved=), or None.  Returns (o, hT or None)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q")
    _check(k, "k", q.dtype, q.shape)
    _check(v, "v", q.dtype, (B, T, H, dv))
    _check(log_g, "log_g", q.dtype, (B, T, H))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_hT else None
    if saved is not None:
        _check(saved, "saved", torch.uint8)
        st = lib.hgrn2_scalar_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(h0), _ptr(o), _ptr(hT),
                                        _ptr(saved), saved.numel(), B, T, H, dk, dv, _dt(q), _stream())
        _raise(st, "hgrn2_scalar_fwd_train")
        return o, hT
    st = lib.hgrn2_scalar_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(h0), _ptr(o), _ptr(hT),
                              B, T, H, dk, dv, _dt(q), _stream())
    _raise(st, "hgrn2_scalar_fwd")
    return o, hT


def scalar_bwd(q, k, v, log_g, dO, h0=None, dhT=None, want_dh0=False, saved=None):
    """Gradients (dq, dk, dv, dlog_g, dh0 or None) of the scalar-decay variant.  saved: the buffer
    a scalar_fwd(..., saved=) on the same inputs filled, or None (the forward then runs again)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q")
    _check(k, "k", q.dtype, q.shape)
    _check(v, "v", q.dtype, (B, T, H, dv))
    _check(log_g, "log_g", q.dtype, (B, T, H))
    _check(dO, "dO", q.dtype, (B, T, H, dv))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    if dhT is not None:
        _check(dhT, "dhT", torch.float32, (B, H, dk, dv))
    dq, dk_, dv_, dg = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(log_g)
    dh0 = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_dh0 else None
    nws = _size_or_raise(lib.hgrn2_scalar_workspace_size(B, T, H, dk, dv, _dt(q), 2 if saved is not None else 1),
                         "hgrn2_scalar_workspace_size")
    ws = _workspace(nws, q.device)
    if saved is not None:
        _check(saved, "saved", torch.uint8)
        st = lib.hgrn2_scalar_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(h0), _ptr(saved), saved.numel(),
                                        _ptr(dO), _ptr(dhT), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(dh0),
                                        B, T, H, dk, dv, _dt(q), _ptr(ws), nws, _stream())
        _raise(st, "hgrn2_scalar_bwd_saved")
        return dq, dk_, dv_, dg, dh0
    st = lib.hgrn2_scalar_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(dq),
                              _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(dh0), B, T, H, dk, dv, _dt(q), _ptr(ws), nws,
                              _stream())
    _raise(st, "hgrn2_scalar_bwd")
    return dq, dk_, dv_, dg, dh0


# ---------------------------------------------------------------- one sequence across GPUs
def state_map(log_f, i):
    """The forward map of a token slice: S_out = Diag(g) S_in + U for every (b, h).

    log_f: [B,T,H,dk]; i: [B,T,H,dv] (same dtype).  Returns (g [B,H,dk], U [B,H,dk,dv]), float32."""
    B, T, H, dk = log_f.shape
    dv = i.shape[-1]
    _check(log_f, "log_f")
    _check(i, "i", log_f.dtype, (B, T, H, dv))
    g = torch.empty((B, H, dk), dtype=torch.float32, device=log_f.device)
    U = torch.empty((B, H, dk, dv), dtype=torch.float32, device=log_f.device)
    _raise(load_library().hgrn2_state_map(_ptr(log_f), _ptr(i), B, T, H, dk, dv, _dt(log_f), _ptr(g), _ptr(U),
                                          _stream()), "hgrn2_state_map")
    return g, U


def state_map_bwd(q, log_f, dO):
    """The backward map of a token slice: dL/dS_in = Diag(g) dL/dS_out + W.

    q, log_f: [B,T,H,dk]; dO: [B,T,H,dv].  Returns (g [B,H,dk], W [B,H,dk,dv]), float32."""
    B, T, H, dk = q.shape
    dv = dO.shape[-1]
    _check(q, "q")
    _check(log_f, "log_f", q.dtype, q.shape)
    _check(dO, "dO", q.dtype, (B, T, H, dv))
    g = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    W = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _raise(load_library().hgrn2_state_map_bwd(_ptr(q), _ptr(log_f), _ptr(dO), B, T, H, dk, dv, _dt(q), _ptr(g),
                                              _ptr(W), _stream()), "hgrn2_state_map_bwd")
    return g, W


def affine_scan(g, M, first: int, count: int, step: int = 1, init=None, out=None):
    """S = init (or 0), then S <- Diag(g_r) S + M_r for r = first, first + step, ... (count maps).

    g: [R,B,H,dk]; M: [R,B,H,dk,dv]; init, out: [B,H,dk,dv] float32 (out may be init)."""
    R, B, H, dk, dv = M.shape
    _check(g, "g", torch.float32, (R, B, H, dk))
    _check(M, "M", torch.float32)
    if init is not None:
        _check(init, "init", torch.float32, (B, H, dk, dv))
    S = out if out is not None else torch.empty((B, H, dk, dv), dtype=torch.float32, device=M.device)
    _check(S, "out", torch.float32, (B, H, dk, dv))
    _raise(load_library().hgrn2_affine_scan(_ptr(g), _ptr(M), R, first, count, step, _ptr(init), _ptr(S), B, H, dk,
                                            dv, _stream()), "hgrn2_affine_scan")
    return S


def device_status() -> int:
    """Synchronises the current stream; returns and clears the device status word."""
    return int(load_library().hgrn2_get_device_status(_stream()))


def selftest_wait_timeout(polls: int = 1000) -> None:
    """Launches the bounded-wait check (see include/hgrn2.h): afterwards device_status()
    returns ERR_TIMEOUT."""
    _raise(load_library().hgrn2_selftest_wait_timeout(polls, _stream()), "hgrn2_selftest_wait_timeout")


def counters(reset: bool = False) -> list[int]:
    """[exact-route (batch, head) passes, tensor-core chunk passes, kernel launches issued]
    since the last reset (synchronises the current stream)."""
    out = (ctypes.c_longlong * 3)()
    _raise(load_library().hgrn2_get_counters(out, 3, int(reset), _stream()), "hgrn2_get_counters")
    return [int(out[0]), int(out[1]), int(out[2])]


class HGRN2Function(torch.autograd.Function):
    """Autograd wrapper: o, hT = HGRN2Function.apply(q, log_f, i, h0, chunk)."""

    @staticmethod
    def forward(ctx, q, log_f, i, h0=None, chunk=64):
        q, log_f, i = q.contiguous(), log_f.contiguous(), i.contiguous()
        h0 = None if h0 is None else h0.contiguous()
        saved = new_saved(q, i.shape[-1])   # chunk states for the backward (None: recompute)
        o, hT = fwd(q, log_f, i, h0, want_hT=True, chunk=chunk, saved=saved)
        ctx.save_for_backward(q, log_f, i, h0, saved)
        ctx.chunk = chunk
        ctx.has_h0 = h0 is not None
        return o, hT

    @staticmethod
    def backward(ctx, dO, dhT):
        q, log_f, i, h0, saved = ctx.saved_tensors
        dq, dlf, di, dh0 = bwd(q, log_f, i, dO.contiguous(), h0,
                               None if dhT is None else dhT.contiguous(),
                               want_dh0=ctx.has_h0, chunk=ctx.chunk, saved=saved)
        return dq, dlf, di, dh0, None


def hgrn2(q, log_f, i, h0=None, chunk=64):
    """Differentiable HGRN2 recurrence: returns (o, hT)."""
    return HGRN2Function.apply(q, log_f, i, h0, chunk)


class ScalarDecayFunction(torch.autograd.Function):
    """Autograd wrapper of the scalar-decay variant: o, hT = ScalarDecayFunction.apply(q, k, v, log_g, h0)."""

    @staticmethod
    def forward(ctx, q, k, v, log_g, h0=None):
        q, k, v, log_g = q.contiguous(), k.contiguous(), v.contiguous(), log_g.contiguous()
        h0 = None if h0 is None else h0.contiguous()
        saved = new_scalar_saved(q, v.shape[-1])   # chunk states for the backward (None: recompute)
        o, hT = scalar_fwd(q, k, v, log_g, h0, want_hT=True, saved=saved)
        ctx.save_for_backward(q, k, v, log_g, h0, saved)
        ctx.has_h0 = h0 is not None
        return o, hT

    @staticmethod
    def backward(ctx, dO, dhT):
        q, k, v, log_g, h0, saved = ctx.saved_tensors
        dq, dk, dv, dg, dh0 = scalar_bwd(q, k, v, log_g, dO.contiguous(), h0,
                                         None if dhT is None else dhT.contiguous(), want_dh0=ctx.has_h0,
                                         saved=saved)
        return dq, dk, dv, dg, dh0


def scalar_decay(q, k, v, log_g, h0=None):
    """Differentiable scalar-decay variant: returns (o, hT)."""
    return ScalarDecayFunction.apply(q, k, v, log_g, h0)
