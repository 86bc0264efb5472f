"""The multi-rank plumbing of bench.py (replicas: no data-path collective) on
CPU: two gloo ranks in separate processes, rendezvous on 127.0.0.1."""
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


def _rank_main(rank, port, times, q, fail_rank):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    try:
        world, r, local = bench.dist_setup(timeout_s=20)
        assert (world, r, local) == (2, rank, rank)
        assert torch.distributed.get_backend() == "gloo"
        bench.barrier(world)
        ms = bench.max_over_ranks(times[rank], world)       # the slowest rank decides
        value = bench.job_throughput(5, world, ms)          # 5 tokens per rank
        if rank == fail_rank:
            raise RuntimeError("rank %d leaves between steps" % rank)
        # the surviving rank's next collective ends with an error, not a hang
        err = None
        if fail_rank is not None:
            try:
                bench.max_over_ranks(1.0, world)
            except Exception as e:  # noqa: BLE001 - any error is the point
                err = type(e).__name__
        q.put((rank, ms, value, err))
    except RuntimeError as e:
        q.put((rank, None, None, str(e)))
    finally:
        if torch.distributed.is_initialized():
            try:
                torch.distributed.destroy_process_group()
            except Exception:  # noqa: BLE001
                pass


def _run(times, fail_rank=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, times, q, fail_rank)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        rank, ms, value, err = q.get(timeout=120)
        out[rank] = (ms, value, err)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode is not None, "a rank did not exit"
    return out


def test_two_ranks_report_the_slowest_rank():
    out = _run([3.0, 4.0])
    for rank in (0, 1):
        ms, value, err = out[rank]
        assert ms == 4.0 and err is None
        assert value == pytest.approx(2 * 5 / 0.004)   # whole job: both ranks' tokens


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    out = _run([1.0, 1.0], fail_rank=1)
    assert "leaves between steps" in out[1][2]
    assert out[0][2] is not None        # rank 0's next collective raised instead of hanging
