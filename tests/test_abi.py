"""The C-ABI library loads and exports every symbol include/hgrn2.h declares.

CPU-only: no call here launches anything or touches a CUDA device (only the
host-side size query and string functions are called).
"""
import ctypes
import os
import re
import subprocess

import pytest

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hgrn2.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hgrn2_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("hgrn2_fwd", "hgrn2_bwd", "hgrn2_step", "hgrn2_workspace_size", "hgrn2_status_string"):
        assert n in names
    assert set(names) == set(L.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(hgrn2_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)


def test_status_strings_and_version(lib):
    for s in range(6):
        assert isinstance(L.status_string(s), str) and L.status_string(s)
    assert L.status_string(99) == "unknown status"
    assert L.version().startswith("hgrn2-b200")


def test_workspace_size_rejects_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    f = lib.hgrn2_workspace_size
    assert f(0, 16, 1, 16, 16, 16, 0, 0) == bad          # B < 1
    assert f(1, -1, 1, 16, 16, 16, 0, 0) == bad          # T < 0
    assert f(1, 16, 1, 257, 16, 16, 0, 0) == bad         # d_k > 256
    assert f(1, 16, 1, 16, 257, 16, 0, 0) == bad         # d_v > 256
    assert f(1, 16, 1, 16, 16, 48, 0, 0) == bad          # chunk not a power of two in [16,128]
    assert f(1, 16, 1, 16, 16, 16, 7, 0) == bad          # unknown dtype
    assert f(1, 16, 1, 16, 16, 16, 0, 0) != bad
    assert f(8, 2048, 16, 128, 128, 64, 1, 1) != bad


def test_bad_arguments_return_errors_before_any_launch(lib):
    # invalid sizes and null pointers are rejected on the host: no CUDA call is made
    vp = ctypes.c_void_p
    st = lib.hgrn2_fwd(None, None, None, None, None, None, 0, 16, 1, 16, 16, 16, 0, None, 0, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_fwd(None, None, None, None, None, None, 1, 16, 1, 16, 16, 16, 0, None, 0, None)
    assert st == L.ERR_INVALID_ARG       # null q
    st = lib.hgrn2_fwd(vp(16), vp(16), vp(16), None, vp(16), None, 1, 16, 1, 16, 16, 24, 0, None, 0, None)
    assert st == L.ERR_UNSUPPORTED       # chunk
    st = lib.hgrn2_fwd(vp(17), vp(16), vp(16), None, vp(16), None, 1, 16, 1, 16, 16, 16, 0, None, 0, None)
    assert st == L.ERR_INVALID_ARG       # misaligned
    st = lib.hgrn2_step(vp(16), vp(16), vp(16), vp(16), vp(16), 1, 1, 16, 6, 0, None)
    assert st == L.ERR_UNSUPPORTED       # d_v not a multiple of 4
    st = lib.hgrn2_bwd(*([None] * 10), 1, 8, 1, 16, 16, 16, 1, None, 0, None)
    assert st == L.ERR_INVALID_ARG


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "linear_attention_hgrn2_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "liboracle" not in txt, fn


def test_saved_size_and_training_pair_argument_checks(lib):
    bad = ctypes.c_size_t(-1).value
    f = lib.hgrn2_saved_size
    # bf16, d = 128: per (b,h) ceil(T/128) bf16 chunk states, one fp32 final state, one flag
    B, T, H = 2, 300, 3
    nt = (T + 127) // 128
    up = lambda x: (x + 255) // 256 * 256
    want = up(B * H * nt * 128 * 128 * 2) + up(B * H * 128 * 128 * 4) + up(B * H * 4)
    assert f(B, T, H, 128, 128, L.BF16) == want
    assert f(B, T, H, 64, 64, L.BF16) == want     # d = 64: the same zero-padded 128 x 128 slots
    assert f(B, T, H, 32, 32, L.BF16) == 0        # exact route: nothing saved
    assert f(B, T, H, 64, 128, L.BF16) == 0
    assert f(B, T, H, 128, 128, L.FP32) == 0
    assert f(B, 0, H, 128, 128, L.BF16) == 0
    assert f(0, T, H, 128, 128, L.BF16) == bad
    vp = ctypes.c_void_p
    # a saved buffer shorter than hgrn2_saved_size is rejected before any launch
    st = lib.hgrn2_fwd_train(vp(16), vp(16), vp(16), None, vp(16), None, vp(256), want - 1,
                             B, T, H, 128, 128, 64, L.BF16, vp(256), 1 << 30, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_bwd_saved(vp(16), vp(16), vp(16), None, None, 0, vp(16), None, vp(16), vp(16), vp(16),
                             None, B, T, H, 128, 128, 64, L.BF16, vp(256), 1 << 30, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_bwd_saved(*([None] * 5), 0, *([None] * 6), 1, 8, 1, 16, 16, 16, 1, None, 0, None)
    assert st == L.ERR_INVALID_ARG       # null inputs (exact route: the buffer is not needed)


def test_step_lb_checks_the_bound_before_any_launch(lib):
    vp = ctypes.c_void_p
    for lb in (-0.5, 1.0, 2.0, float("nan")):
        st = lib.hgrn2_step_lb(vp(16), vp(16), vp(16), ctypes.c_float(lb), vp(16), vp(16), 1, 1, 16, 16, 0, None)
        assert st == L.ERR_INVALID_ARG, lb


def test_packed_sequence_sizes_and_argument_checks(lib):
    bad = ctypes.c_size_t(-1).value
    up = lambda x: (x + 255) // 256 * 256
    nseq, T, H = 5, 700, 3
    # chunk-state slots: sequence s's chunk n sits at ((cu[s] >> 7) + s + n) * H + h, so
    # (T >> 7) + nseq slot rows cover any packing of T tokens into nseq sequences
    slots = ((T >> 7) + nseq) * H
    # + final states, flags, and the launch order of the sequences
    want = up(slots * 128 * 128 * 2) + up(nseq * H * 128 * 128 * 4) + up(nseq * H * 4) + up(nseq * 4)
    assert lib.hgrn2_saved_size_varlen(nseq, T, H, 128, 128, L.BF16) == want
    assert lib.hgrn2_saved_size_varlen(nseq, T, H, 64, 64, L.BF16) == want
    assert lib.hgrn2_saved_size_varlen(nseq, T, H, 32, 32, L.BF16) == 0
    assert lib.hgrn2_saved_size_varlen(nseq, 0, H, 128, 128, L.BF16) == 0
    assert lib.hgrn2_saved_size_varlen(0, T, H, 128, 128, L.BF16) == bad
    ws = lib.hgrn2_workspace_size_varlen(nseq, T, H, 128, 128, 64, L.BF16)
    assert ws == up(nseq * H * 128 * 4) + up(nseq * H * 4) + up(nseq * 4)
    assert lib.hgrn2_workspace_size_varlen(nseq, T, H, 128, 128, 48, L.BF16) == bad
    vp = ctypes.c_void_p
    args = (nseq, T, H, 128, 128, 64, L.BF16)
    # null or misaligned cu_seqlens, a short saved buffer: rejected before any launch
    for cu in (None, vp(20)):
        st = lib.hgrn2_fwd_varlen(vp(16), vp(16), vp(16), None, vp(16), None, cu, *args, None, 0,
                                  vp(256), ws, None)
        assert st == L.ERR_INVALID_ARG
        st = lib.hgrn2_bwd_varlen(vp(16), vp(16), vp(16), None, None, 0, vp(16), None, vp(16), vp(16),
                                  vp(16), None, cu, *args, vp(256), ws, None)
        assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_fwd_varlen(vp(16), vp(16), vp(16), None, vp(16), None, vp(16), *args, vp(256), want - 1,
                              vp(256), ws, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_bwd_varlen(vp(16), vp(16), vp(16), None, vp(256), want - 1, vp(16), None, vp(16), vp(16),
                              vp(16), None, vp(16), *args, vp(256), ws, None)
    assert st == L.ERR_INVALID_ARG
    # workspace shorter than hgrn2_workspace_size_varlen
    st = lib.hgrn2_fwd_varlen(vp(16), vp(16), vp(16), None, vp(16), None, vp(16), *args, None, 0,
                              vp(256), ws - 1, None)
    assert st == L.ERR_INVALID_ARG


def test_step_bwd_argument_checks_before_any_launch(lib):
    vp = ctypes.c_void_p
    B, H, dk, dv = 2, 2, 16, 16
    n = B * H * dk * dv * 4
    base = [vp(256), vp(256), vp(256), vp(4096)]   # q, log_f, i, S
    # dS_prev overlapping dS without being it
    st = lib.hgrn2_step_bwd(*base, vp(256), vp(1 << 20), vp((1 << 20) + 16), vp(256), vp(256), vp(256),
                            B, H, dk, dv, L.FP32, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_step_bwd(*base, vp(256), vp(1 << 20), vp((1 << 20) + n - 16), vp(256), vp(256), vp(256),
                            B, H, dk, dv, L.FP32, None)
    assert st == L.ERR_INVALID_ARG
    # null outputs, dv not a multiple of 4, misaligned state
    st = lib.hgrn2_step_bwd(*base, vp(256), None, None, None, vp(256), vp(256), B, H, dk, dv, L.FP32, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_step_bwd(*base, vp(256), None, None, vp(256), vp(256), vp(256), B, H, dk, 6, L.FP32, None)
    assert st == L.ERR_UNSUPPORTED
    st = lib.hgrn2_step_bwd(vp(256), vp(256), vp(256), vp(4100), vp(256), None, None, vp(256), vp(256), vp(256),
                            B, H, dk, dv, L.FP32, None)
    assert st == L.ERR_INVALID_ARG
    for lb in (-0.1, 1.0, float("nan")):
        st = lib.hgrn2_step_lb_bwd(vp(256), vp(256), vp(256), ctypes.c_float(lb), vp(4096), vp(256), None, None,
                                   vp(256), vp(256), vp(256), B, H, dk, dv, L.FP32, None)
        assert st == L.ERR_INVALID_ARG, lb


def test_workspace_size_of_the_backward_with_saved_states(lib):
    f = lib.hgrn2_workspace_size
    bad = ctypes.c_size_t(-1).value
    up = lambda x: (x + 255) // 256 * 256
    B, T, H = 2, 300, 3
    assert f(B, T, H, 64, 64, 64, L.BF16, 2) <= f(B, T, H, 64, 64, 64, L.BF16, 1)
    # d = 64 without saved states: room for the chunk states and an o scratch on top
    extra = lib.hgrn2_saved_size(B, T, H, 64, 64, L.BF16) + up(B * T * H * 64 * 2)
    assert f(B, T, H, 64, 64, 64, L.BF16, 1) == f(B, T, H, 64, 64, 64, L.BF16, 2) + extra
    # d = 128 with saved states and few (b,h): the backward runs in sequence segments, cut as the
    # forward cuts them (148 // (B*H) per pair, at most one per chunk), and keeps every segment's
    # backward map (128 x 128 + 128 floats) and the quarter sums of |W| per row (4 x 128 floats)
    def nseg(B, T, H):
        ntiles = (T + 127) // 128
        ns = min(max(1, 148 // (B * H)), ntiles)
        tps = (ntiles + ns - 1) // ns
        return (ntiles + tps - 1) // tps
    # Without saved states and with segments, the backward runs the training forward into its
    # workspace and then the saved-state backward: room for both, the saved buffer and an o scratch.
    for (B, T, H) in ((2, 300, 3), (1, 32768, 8), (8, 2048, 16)):
        ns = nseg(B, T, H)
        seg = up(B * H * ns * (128 * 128 + 128 + 512) * 4) if ns > 1 else 0
        base = up(B * H * 128 * 4) + up(B * H * 4)   # rowsum(dhT * hT), exact-route flags
        assert f(B, T, H, 128, 128, 64, L.BF16, 2) == base + seg, (B, T, H)
        if ns > 1:
            extra = up(lib.hgrn2_saved_size(B, T, H, 128, 128, L.BF16)) + up(B * T * H * 128 * 2) + \
                f(B, T, H, 128, 128, 64, L.BF16, 0)
            assert f(B, T, H, 128, 128, 64, L.BF16, 1) == base + seg + extra, (B, T, H)
        else:
            assert f(B, T, H, 128, 128, 64, L.BF16, 1) == base, (B, T, H)
    assert nseg(8, 2048, 16) == 1 and nseg(1, 32768, 8) == 18
    # the forward with segments: per segment its U (128 x 128), g, the first chunk's total decay and
    # the row sums of |U| (3 x 128 floats), the first chunk's bf16 q e^{b} (128 x 128); then the
    # per-pair finished-segment counts
    for (B, T, H) in ((2, 300, 3), (1, 32768, 8), (8, 2048, 16), (4, 2048, 8)):
        ns = nseg(B, T, H)
        fseg = up(B * H * ns * ((128 * 128 + 3 * 128) * 4 + 128 * 128 * 2) + B * H * 4) if ns > 1 else 0
        assert f(B, T, H, 128, 128, 64, L.BF16, 0) == up(B * H * 4) + fseg, (B, T, H)
    assert f(B, T, H, 64, 64, 64, L.BF16, 3) == bad
    assert f(B, T, H, 64, 64, 64, L.BF16, -1) == bad


def test_selftest_checks_its_poll_count_before_any_launch(lib):
    assert lib.hgrn2_selftest_wait_timeout(0, None) == L.ERR_INVALID_ARG
    assert lib.hgrn2_selftest_wait_timeout((1 << 24) + 1, None) == L.ERR_INVALID_ARG


def test_scalar_decay_argument_checks_before_any_launch(lib):
    vp = ctypes.c_void_p
    bad = ctypes.c_size_t(-1).value
    up = lambda x: (x + 255) // 256 * 256
    ws = lib.hgrn2_scalar_workspace_size
    assert ws(0, 8, 4, 16, 16, L.FP32, 1) == bad
    assert ws(2, 8, 3, 16, 16, L.FP32, 3) == bad
    assert ws(2, 8, 3, 16, 16, L.FP32, 0) == 0                      # the forward needs none
    # exact route: <dhT, hT> per (b,h) and q . dq per token, fp32
    assert ws(2, 8, 3, 16, 16, L.FP32, 1) == up(4 * 2 * 3) + up(4 * 2 * 8 * 3)
    B, T, H = 2, 300, 3   # tensor-core route: + the saved chunk states and an o scratch, unless given
    saved = lib.hgrn2_saved_size(B, T, H, 128, 128, L.BF16)
    assert lib.hgrn2_scalar_saved_size(B, T, H, 128, 128, L.BF16) == saved
    assert lib.hgrn2_scalar_saved_size(B, T, H, 32, 32, L.BF16) == 0
    assert ws(B, T, H, 128, 128, L.BF16, 2) == up(4 * B * H) + up(4 * B * T * H)
    assert ws(B, T, H, 128, 128, L.BF16, 1) == ws(B, T, H, 128, 128, L.BF16, 2) + saved + up(B * T * H * 128 * 2)
    # a saved buffer shorter than the saved size: rejected before any launch
    st = lib.hgrn2_scalar_fwd_train(vp(16), vp(16), vp(16), vp(16), None, vp(16), None, vp(256), saved - 1,
                                    B, T, H, 128, 128, L.BF16, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_scalar_bwd_saved(vp(16), vp(16), vp(16), vp(16), None, vp(256), saved - 1, vp(16), None,
                                    vp(16), vp(16), vp(16), vp(16), None, B, T, H, 128, 128, L.BF16, vp(256),
                                    1 << 30, None)
    assert st == L.ERR_INVALID_ARG
    f = lib.hgrn2_scalar_fwd
    assert f(vp(16), vp(16), vp(16), vp(16), None, vp(16), None, 1, 8, 1, 256, 16, L.FP32, None) == L.ERR_UNSUPPORTED
    assert f(None, vp(16), vp(16), vp(16), None, vp(16), None, 1, 8, 1, 16, 16, L.FP32, None) == L.ERR_INVALID_ARG
    assert f(vp(18), vp(16), vp(16), vp(16), None, vp(16), None, 1, 8, 1, 16, 16, L.FP32, None) == L.ERR_INVALID_ARG
    g = lib.hgrn2_scalar_bwd
    # workspace missing or short
    args = [vp(16)] * 4 + [None, vp(16), None] + [vp(16)] * 4 + [None]
    assert g(*args, 2, 8, 3, 16, 16, L.BF16, None, 0, None) == L.ERR_INVALID_ARG
    assert g(*args, 2, 8, 3, 16, 16, L.BF16, vp(256), 255, None) == L.ERR_INVALID_ARG
    assert g(*args, 2, 300, 3, 128, 128, L.BF16, vp(256), 256, None) == L.ERR_INVALID_ARG   # no room for states


def test_wide_heads_sizes(lib):
    # heads wider than 128 run as blocks of <= 128: the workspace holds the column copies, the
    # blocks' partial outputs, their state blocks and the block calls' own workspace; the saved
    # buffer that of one call over all blocks (equal blocks) or one region per block pair
    bad = ctypes.c_size_t(-1).value
    B, T, H = 2, 300, 3
    ws = lib.hgrn2_workspace_size
    for dk, dv in ((256, 256), (192, 160), (100, 256), (256, 64)):
        for want in (0, 1, 2):
            assert ws(B, T, H, dk, dv, 64, L.BF16, want) not in (bad, 0)
            assert ws(B, T, H, dk, dv, 64, L.FP32, want) not in (bad, 0)
    one = lib.hgrn2_saved_size(B, T, H, 128, 128, L.BF16)
    up = lambda x: (x + 255) // 256 * 256
    # equal blocks run as one call over H * (blocks per head) heads
    assert lib.hgrn2_saved_size(B, T, H, 256, 256, L.BF16) == lib.hgrn2_saved_size(B, T, 4 * H, 128, 128, L.BF16)
    assert lib.hgrn2_saved_size(B, T, H, 256, 128, L.BF16) == lib.hgrn2_saved_size(B, T, 2 * H, 128, 128, L.BF16)
    assert lib.hgrn2_saved_size(B, T, H, 64, 256, L.BF16) == 0   # 64 x 128 blocks: exact route
    # blocks (0,0) 128 x 128 and (1,1) 64 x 64 take the tensor cores, (0,1) and (1,0) do not
    assert lib.hgrn2_saved_size(B, T, H, 192, 192, L.BF16) == up(one) + up(lib.hgrn2_saved_size(B, T, H, 64, 64, L.BF16))
    assert lib.hgrn2_saved_size(B, T, H, 256, 256, L.FP32) == 0
    # packed sequences and the decode step stay at <= 128
    assert lib.hgrn2_workspace_size_varlen(2, 300, H, 256, 256, 64, L.BF16) == bad
    assert lib.hgrn2_saved_size_varlen(2, 300, H, 256, 256, L.BF16) == bad
    vp = ctypes.c_void_p
    st = lib.hgrn2_step(vp(256), vp(256), vp(256), vp(4096), vp(256), 1, 1, 256, 256, L.FP32, None)
    assert st == L.ERR_UNSUPPORTED


def test_no_fallback_without_the_library_or_a_device():
    # a fresh process: the library handle is cached per process.  A missing .so raises at load
    # time, and a call on host tensors raises instead of computing anything on the CPU.
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import linear_attention_hgrn2_b200 as L, torch\n"
        "try:\n"
        "    L.load_library('/nonexistent/libhgrn2.so'); print('loaded')\n"
        "except ImportError:\n"
        "    print('missing raises')\n"
        "L._lib = None\n"
        "q = torch.zeros(1, 4, 1, 8, dtype=torch.bfloat16)\n"
        "try:\n"
        "    L.fwd(q, q, q); print('computed on host')\n"
        "except Exception as e:\n"
        "    print('host tensors raise', type(e).__name__)\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.strip().splitlines()
    assert lines[0] == "missing raises"
    assert lines[1].startswith("host tensors raise"), lines


def test_wide_heads_reject_bad_arguments_before_any_launch(lib):
    # the wide-head path checks like every other call before it launches anything; on a machine
    # without a GPU a launch would surface as ERR_CUDA, so ERR_INVALID_ARG shows none was made
    vp = ctypes.c_void_p
    B, T, H, dk, dv = 1, 16, 1, 256, 256
    need = lib.hgrn2_workspace_size(B, T, H, dk, dv, 64, L.BF16, 0)
    assert need > 0
    st = lib.hgrn2_fwd(vp(256), vp(256), vp(256), None, vp(256), None, B, T, H, dk, dv, 64, L.BF16, vp(256),
                       need - 1, None)
    assert st == L.ERR_INVALID_ARG       # workspace one byte short
    st = lib.hgrn2_fwd(None, vp(256), vp(256), None, vp(256), None, B, T, H, dk, dv, 64, L.BF16, vp(256), need, None)
    assert st == L.ERR_INVALID_ARG       # q missing
    st = lib.hgrn2_fwd(vp(256), vp(256), vp(258), None, vp(256), None, B, T, H, dk, dv, 64, L.BF16, vp(256), need,
                       None)
    assert st == L.ERR_INVALID_ARG       # i not 16-byte aligned
    needb = lib.hgrn2_workspace_size(B, T, H, dk, dv, 64, L.BF16, 1)
    st = lib.hgrn2_bwd(vp(256), vp(256), vp(256), None, vp(256), None, vp(256), vp(256), vp(256), None,
                       B, T, H, dk, dv, 64, L.BF16, vp(256), needb - 1, None)
    assert st == L.ERR_INVALID_ARG
    st = lib.hgrn2_fwd(vp(256), vp(256), vp(256), None, vp(256), None, B, T, H, 257, dv, 64, L.BF16, vp(256), need,
                       None)
    assert st == L.ERR_UNSUPPORTED       # wider than 256


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: a C99 program includes the header, links the library and calls it
    # (host-only calls: sizes, version, an argument error)
    import shutil
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.isdir(cuda_inc):
        pytest.skip("no C compiler or CUDA headers")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "linear_attention_hgrn2_b200")
    src = tmp_path / "t.c"
    src.write_text(
        "#include <stdio.h>\n#include \"hgrn2.h\"\n"
        "int main(void) {\n"
        "    size_t ws = hgrn2_workspace_size(8, 2048, 16, 128, 128, 64, HGRN2_BF16, 1);\n"
        "    hgrn2_status st = hgrn2_fwd(NULL, NULL, NULL, NULL, NULL, NULL, 0, 16, 1, 16, 16, 16, HGRN2_FP32,\n"
        "                                NULL, 0, NULL);\n"
        "    printf(\"%s|%zu|%d|%s\\n\", hgrn2_version(), ws, (int)st, hgrn2_status_string(st));\n"
        "    return 0;\n}\n")
    exe = tmp_path / "t"
    cc = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                         "-I", cuda_inc, str(src), "-L", pkg, "-lhgrn2", f"-Wl,-rpath,{pkg}", "-o", str(exe)],
                        capture_output=True, text=True, timeout=120)
    assert cc.returncode == 0, cc.stderr[-2000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr[-2000:]
    version, ws, st, msg = run.stdout.strip().split("|")
    assert version.startswith("hgrn2-b200") and int(ws) > 0
    assert int(st) == L.ERR_INVALID_ARG and msg


@pytest.mark.parametrize("dt,d,limit", [(L.BF16, 128, 2032), (L.FP32, 128, 2048), (L.BF16, 64, 4032)])
def test_noalloc_size_limit_boundary(lib, dt, d, limit):
    # the allocation-free backward needs hgrn2_workspace_size(..., want_bwd = 2) bytes of its fixed
    # scratch: B*H = limit fits exactly, limit + 1 does not and is refused on the host, before any
    # launch (so this runs without a GPU; the accepted size is only sized, never called)
    cap = 1 << 20
    f = lib.hgrn2_workspace_size
    assert f(1, 64, limit, d, d, 64, dt, 2) <= cap
    assert f(1, 64, limit + 1, d, d, 64, dt, 2) > cap
    vp = ctypes.c_void_p(16)
    st = lib.hgrn2_bwd_noalloc(vp, vp, vp, None, vp, None, vp, vp, vp, None, 1, 64, limit + 1, d, d, 64, dt, None)
    assert st == L.ERR_UNSUPPORTED


def test_sequence_parallel_entry_points_check_their_arguments(lib):
    # host-side refusals, before any launch
    vp = ctypes.c_void_p
    a, b = vp(1 << 20), vp(1 << 24)   # two aligned, disjoint stand-in addresses (never dereferenced)
    # state maps: key dims above 128, unknown dtype, null outputs, misaligned pointers
    assert lib.hgrn2_state_map(a, a, 1, 8, 1, 129, 16, L.FP32, a, b, None) == L.ERR_UNSUPPORTED
    assert lib.hgrn2_state_map(a, a, 1, 8, 1, 16, 16, 7, a, b, None) == L.ERR_INVALID_ARG
    assert lib.hgrn2_state_map(a, a, 1, 8, 1, 16, 16, L.FP32, None, b, None) == L.ERR_INVALID_ARG
    assert lib.hgrn2_state_map_bwd(None, a, a, 1, 8, 1, 16, 16, L.FP32, a, b, None) == L.ERR_INVALID_ARG
    assert lib.hgrn2_state_map(vp((1 << 20) + 4), a, 1, 8, 1, 16, 16, L.FP32, a, b, None) == L.ERR_INVALID_ARG
    # scan: maps outside [0, R), a step other than +-1, an output overlapping the maps
    f = lib.hgrn2_affine_scan
    assert f(a, b, 4, 3, 2, 1, None, vp(1 << 28), 1, 1, 16, 16, None) == L.ERR_INVALID_ARG   # maps 3, 4
    assert f(a, b, 4, 1, 3, -1, None, vp(1 << 28), 1, 1, 16, 16, None) == L.ERR_INVALID_ARG  # maps 1, 0, -1
    assert f(a, b, 4, 0, 2, 2, None, vp(1 << 28), 1, 1, 16, 16, None) == L.ERR_INVALID_ARG
    assert f(a, b, 4, 0, 2, 1, None, b, 1, 1, 16, 16, None) == L.ERR_INVALID_ARG            # S on M
    assert f(a, b, 4, 0, 2, 1, None, None, 1, 1, 16, 16, None) == L.ERR_INVALID_ARG          # no output
