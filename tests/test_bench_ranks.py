"""The multi-process side of bench.py, on CPU: two `gloo` ranks.

bench.py --gpus N runs N independent replicas (one problem per GPU, no
data-path collective).  What the ranks do share is the timing: a barrier
around the timed region, the slowest rank's time (max over ranks), and the
whole-job throughput computed from it.  The reference arm runs on rank 0 only.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, lr = bench.dist_env()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        slowest = bench.max_over_ranks(1.0 + rank)   # rank 1 is the slower one
        # two replicas of 7 tokens per step, 10 steps, over the slowest rank's 2.0 s
        tput = bench.throughput(7, 10, w, slowest)

        class Args:
            steps, warmup = 1, 0
        ref = bench.run_reference(Args, r, w) if r != 0 else "rank0-skipped"
        bench.barrier()
        out.put((r, w, lr, slowest, tput, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, w, lr, slowest, tput, ref) in enumerate(res):
        assert (r, w, lr) == (rank, world, rank)
        assert slowest == 2.0                      # both ranks see the max
        assert tput == pytest.approx(7 * 10 * 2 / 2.0)
    # the reference arm does no work off rank 0
    assert res[1][5] is None


def test_single_process_helpers_are_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    bench.barrier()   # no process group: a no-op
    assert bench.throughput(1, 100, 1, 0.5) == 200.0
