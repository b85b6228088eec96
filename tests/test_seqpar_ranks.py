"""Sequence parallelism across ranks: the host logic, on CPU with two and three gloo ranks.

Each rank holds one contiguous slice of every (batch, head) sequence.  The library's
sequence-parallel driver (linear_attention_hgrn2_b200.seqpar) computes the slice's state maps,
all-gathers them over the process group, scans them in rank order (forward) and reverse rank
order (backward), and runs the slice from its boundary states.  Here the compute steps are the
fp64 oracle and a NumPy scan (the ``ops`` hook), so the test checks what the driver itself does
- slicing, the order of the gathered maps, the scan ranges and directions, the boundary states,
which rank returns dh0 - against the oracle run over the whole sequence.  The kernels behind the
same steps are checked on the GPU in test_seqpar.py.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The compute steps of a sequence-parallel pass on the host, in fp64 (test only)."""

    @staticmethod
    def state_map(log_f, i):
        import oracle
        lf = log_f.double().numpy()
        _, U = oracle.fwd(np.zeros_like(lf), lf, i.double().numpy())        # the state from zero
        return torch.from_numpy(np.exp(lf.sum(axis=1))), torch.from_numpy(U)

    @staticmethod
    def state_map_bwd(q, log_f, dO):
        import oracle
        lf = log_f.double().numpy()
        # dL/dS_in with nothing leaving the slice (dhT = 0): the slice's own map W; it does not
        # depend on i or on the state entering the slice
        dh0 = oracle.bwd(q.double().numpy(), lf, np.zeros_like(dO.double().numpy()), dO.double().numpy())[3]
        return torch.from_numpy(np.exp(lf.sum(axis=1))), torch.from_numpy(dh0)

    @staticmethod
    def affine_scan(g, M, first, count, step, init=None):
        S = np.zeros(M.shape[1:]) if init is None else init.double().numpy().copy()
        r = first
        for _ in range(count):
            S = g[r].double().numpy()[..., None] * S + M[r].double().numpy()
            r += step
        return torch.from_numpy(S)

    @staticmethod
    def fwd(q, log_f, i, h0, saved=None, chunk=64):
        import oracle
        o, hT = oracle.fwd(q.double().numpy(), log_f.double().numpy(), i.double().numpy(),
                           None if h0 is None else h0.double().numpy())
        return torch.from_numpy(o), torch.from_numpy(hT)

    @staticmethod
    def bwd(q, log_f, i, dO, h0, dhT, want_dh0, saved=None, chunk=64):
        import oracle
        n = lambda t: None if t is None else t.double().numpy()
        return tuple(torch.from_numpy(a) for a in oracle.bwd(n(q), n(log_f), n(i), n(dO), n(h0), n(dhT)))


def _bounds(T, world):
    # unequal slices: rank r gets T // world tokens plus one of the remainder's, in order
    base, rem = divmod(T, world)
    lens = [base + (1 if r < rem else 0) for r in range(world)]
    return np.concatenate([[0], np.cumsum(lens)]).astype(int)


def _worker(rank, world, port, T, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from linear_attention_hgrn2_b200 import inputs as I
    from linear_attention_hgrn2_b200 import seqpar
    from test_seqpar_ranks import OracleOps
    inp = I.make_inputs(2, T, 3, 4, 5, torch.float32, 0.3, seed=71, h0_sigma=0.5, with_dO=True, dhT_sigma=0.5)
    b = _bounds(T, world)
    sl = lambda t: t[:, b[rank]:b[rank + 1]].contiguous()
    q, lf, x, dO = (sl(inp[k]) for k in ("q", "log_f", "i", "dO"))
    o, hT, ctx = seqpar.forward(q, lf, x, inp["h0"], ops=OracleOps)
    dq, dlf, di, dh0 = seqpar.backward(q, lf, x, dO, ctx, dhT=inp["dhT"], ops=OracleOps)
    q_out.put((rank, o.numpy(), hT.numpy(), dq.numpy(), dlf.numpy(), di.numpy(),
               None if dh0 is None else dh0.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 37), (3, 50)])
def test_sequence_parallel_ranks_match_the_whole_sequence(world, T):
    import oracle
    sys.path.insert(0, ROOT)
    from linear_attention_hgrn2_b200 import inputs as I
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_out.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = I.make_inputs(2, T, 3, 4, 5, torch.float32, 0.3, seed=71, h0_sigma=0.5, with_dO=True, dhT_sigma=0.5)
    n = lambda t: t.double().numpy()
    o, hT = oracle.fwd(n(inp["q"]), n(inp["log_f"]), n(inp["i"]), n(inp["h0"]))
    dq, dlf, di, dh0 = oracle.bwd(n(inp["q"]), n(inp["log_f"]), n(inp["i"]), n(inp["dO"]), n(inp["h0"]),
                                  n(inp["dhT"]))
    b = _bounds(T, world)
    for r, o_r, hT_r, dq_r, dlf_r, di_r, dh0_r in res:
        s = slice(b[r], b[r + 1])
        np.testing.assert_allclose(o_r, o[:, s], rtol=0, atol=1e-12)
        np.testing.assert_allclose(hT_r, hT, rtol=0, atol=1e-12)   # every rank: the whole sequence's hT
        np.testing.assert_allclose(dq_r, dq[:, s], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dlf_r, dlf[:, s], rtol=0, atol=1e-12)
        np.testing.assert_allclose(di_r, di[:, s], rtol=0, atol=1e-12)
        if r == 0:
            np.testing.assert_allclose(dh0_r, dh0, rtol=0, atol=1e-12)
        else:
            assert dh0_r is None
