"""Failure reporting on the GPU without a fault.

Every wait inside the library's kernels is bounded; a wait that gives up records
HGRN2_ERR_TIMEOUT in the device status word and its kernel exits normally.  The check kernel
behind hgrn2_selftest_wait_timeout waits, through the same bounded-wait helper, on a barrier
that nothing arrives at: the host must read HGRN2_ERR_TIMEOUT, the word must clear on reading,
and the context must stay usable (the next call computes correct results).
"""
import pytest
import torch

import linear_attention_hgrn2_b200 as L
from linear_attention_hgrn2_b200 import inputs as I
from parity_util import err, np64, oracle_heads, to_cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_timeout_and_the_context_stays_usable(cuda):
    assert L.device_status() == L.OK
    L.selftest_wait_timeout(1000)
    assert L.device_status() == L.ERR_TIMEOUT
    assert L.device_status() == L.OK   # reading clears the word
    inp = I.make_inputs(1, 300, 2, 128, 128, torch.bfloat16, 0.9, seed=801, h0_sigma=0.1)
    g = to_cuda(inp)
    o, hT = L.fwd(g["q"], g["log_f"], g["i"], g["h0"], want_hT=True)
    assert L.device_status() == L.OK
    ref = oracle_heads(inp, [(0, 0), (0, 1)])
    for n, h in enumerate((0, 1)):
        assert err(np64(o[0, :, h]), ref["o"][n], torch.bfloat16) <= 2e-2
        assert err(np64(hT[0, h]), ref["hT"][n], torch.bfloat16) <= 2e-2
