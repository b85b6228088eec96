"""The N > 1 host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

One process per GPU in the real run (NCCL); the data path has no collective, so what needs
checking is the host side: rendezvous, barriers, the max over ranks of the timed interval,
the whole-job value, the per-rank inputs, and that only rank 0 reports (the reference arm
does no work on other ranks).
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(backend="gloo")
    bench.barrier(w)
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w)          # rank 1 is the slower one
    value = bench.whole_job_value(8 * 2048, 4, ms, w)
    from linear_attention_hgrn2_b200 import inputs as I
    inp = I.make_inputs(1, 8, 1, 4, 4, __import__("torch").float32, 0.5, seed=bench.rank_seed(r))
    ref_ret = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), w, r) if r != 0 else None
    q.put((r, w, ms, value, float(inp["q"].sum()), ref_ret))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_time_and_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for r, w, ms, value, _, _ in res:
        assert w == world
        assert ms == 15.0                                   # the max over ranks, on every rank
        assert value == pytest.approx(world * 8 * 2048 * 4 / 0.015)
    assert res[0][4] != res[1][4]                           # each rank draws its own batch
    assert res[1][5] is None                                # reference arm: rank 1 returns without work
