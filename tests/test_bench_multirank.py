"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The layer has no exchange step, so N GPUs run N replicas; what the ranks share
is the timing protocol: a barrier on both sides of the timed region and the
maximum of the per-rank device times.  The reference arm runs on rank 0 only."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    w, r, local = bench._dist_init()
    try:
        assert (w, r, local) == (world, rank, rank)
        assert dist.get_backend() == "gloo"
        bench._barrier(w)
        t = bench._max_over_ranks(10.0 + 5.0 * rank, w)  # each rank's own "elapsed time"
        bench._barrier(w)

        class A:
            steps, warmup, gpus = 1, 0, world

        bench.run_reference(A, w, r) if r != 0 else None  # non-zero ranks leave without work
        out.put((rank, t))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = dict(out.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}
