"""bench.py's multi-rank plumbing on the CPU: two gloo ranks set up the process
group from the launcher's environment, take the element-wise maximum of their
timings and meet at a barrier (the code the GPU run uses over NCCL)."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    bench = _bench()
    w, r, local = bench.dist_setup("gloo")
    assert (w, r, local) == (world, rank, rank)
    got = bench.max_over_ranks([1.5 + rank, 10.0 - rank, 3.0 * rank], w)
    bench.barrier(w)
    out[rank] = got
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_of_their_timings():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        assert out[r] == [2.5, 10.0, 3.0]


def test_one_rank_needs_no_process_group():
    bench = _bench()
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup("gloo") == (1, 0, 0)
    assert bench.max_over_ranks([4.0, 2.0], 1) == [4.0, 2.0]
