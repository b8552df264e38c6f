"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

bench.py --gpus N runs N independent replicas (the decode has no exchange
step), one process per GPU, and reports the slowest rank's step time and the
whole job's bytes over it.  This checks rendezvous, the max over ranks and the
barrier with two gloo ranks, which is what the NCCL run does on GPUs.
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


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    got_ws, got_rank, _ = bench.dist_setup("gloo")
    t_mine = 1e-3 * (1 + got_rank)            # rank r "took" (r + 1) ms
    t_max = bench.max_over_ranks(t_mine, got_ws, device="cpu")
    bench.barrier(got_ws)
    out.put((got_rank, got_ws, t_max, bench.job_gbs(75497472, t_max, got_ws)))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, out)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for _, got_ws, t_max, gbs in res:
        assert got_ws == 2
        assert t_max == pytest.approx(2e-3)        # the slower rank's time on both ranks
        assert gbs == pytest.approx(2 * 75497472 / 2e-3 / 1e9)


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1) == 0.5
    assert bench.job_gbs(1e9, 1.0, 1) == pytest.approx(1.0)
