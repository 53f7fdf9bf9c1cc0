"""The multi-process plumbing of bench.py on the host: two gloo ranks started
like torchrun's workers (RANK / WORLD_SIZE / MASTER_* in the environment).
Each rank runs its own problem (independent replicas, no collective on the data
path); the step time reported is the maximum over ranks, and every rank takes
the same collective steps in the same order."""

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


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    w, r, _ = bench.dist_setup(backend="gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # a per-rank "step time": the slowest rank's must be reported by everyone
    got = bench.max_over_ranks(1.0 + 0.25 * rank, w)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((rank, got))


@pytest.mark.parametrize("world", [2])
def test_step_time_is_the_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out.get(timeout=10) for _ in range(world))
    assert res == {r: 1.0 + 0.25 * (world - 1) for r in range(world)}


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
