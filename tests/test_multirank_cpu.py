"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun
would launch them (RANK / WORLD_SIZE / MASTER_ADDR 127.0.0.1), run the
barrier, the max-over-ranks time and the whole-job rate, and the reference
arm's rank gating (rank 0 alone runs the oracle).  The forward itself is a
replica per GPU with no collective on the data path, so this is all the
multi-GPU logic there is."""

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
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    r, local, w = bench._dist_setup(world)
    assert (r, local, w) == (rank, rank, world)
    assert dist.get_backend() == "gloo"
    bench._barrier(w)
    # each rank times a different region; every rank must see the slowest
    ms = bench._max_over_ranks(10.0 + rank, w)
    rate = bench._job_rate(w, 4096, ms)
    # the reference arm: rank 0 alone runs it, the others return at once
    if rank != 0:
        line, w2 = bench.run_reference(None)
        assert line is None and w2 == world
    bench._barrier(w)
    dist.destroy_process_group()
    out.put((rank, ms, rate))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, rate in got:
        assert ms == 11.0                                   # the max over both ranks
        assert rate == pytest.approx(2 * 4096 / 11.0e-3)    # both ranks' tokens / slowest time
