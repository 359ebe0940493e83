"""Host logic of the multi-GPU benchmark path on the CPU: two ranks on the
gloo backend (one process each, as torchrun would start them) check that
every rank draws its own batch, that the reported time is the slowest rank's
and that the whole-job rate counts the units of every rank."""
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


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo")
    assert (w, r) == (world, rank)
    # each rank's own timing: the slowest (rank 1) must be reported everywhere
    ms_local = 10.0 + 5.0 * rank
    ms_max = bench.max_over_ranks(ms_local, w)
    bench.barrier(w)
    seed = bench.rank_seed(2, rank)
    rate = bench.whole_job_rate(1000, w, ms_max)
    with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
        f.write("%r %r %r\n" % (ms_max, seed, rate))
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    rows = [open(tmp_path / ("rank%d.txt" % r)).read().split() for r in range(world)]
    ms = [float(x[0]) for x in rows]
    seeds = [int(x[1]) for x in rows]
    rates = [float(x[2]) for x in rows]
    assert ms == [15.0, 15.0]                      # max over ranks, seen by every rank
    assert len(set(seeds)) == world                # distinct batches per rank
    assert rates[0] == pytest.approx(2 * 1000 / 0.015)  # units of both ranks / slowest time
