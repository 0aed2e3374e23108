"""The multi-GPU host logic of bench.py on CPU: two ranks over gloo (the GPU
job uses NCCL with the same calls).  Each rank runs its own replica of the
step; the job's time is the slowest rank's, its value the bytes of all ranks
over that time; the reference arm runs on rank 0 only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.world_info() == (world, rank, rank)
        # rank r took (r + 1) ms per step and 10 - r ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], dist, "cpu")
        value = bench.job_value(1.0e9, world, got[0])
        # the reference arm: ranks other than 0 return at once and print nothing
        buf = io.StringIO()
        if rank != 0:
            class A:
                fmt, batch, steps, warmup, gpus, model, layers = "q1g128", 1, 1, 0, world, "qwen3-8b", 36
            with redirect_stdout(buf):
                assert bench.run_reference(A()) == 0
        dist.barrier()
        out.put((rank, got, value, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_job_value():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value, printed in res:
        assert got == [2.0, 10.0]            # the slowest rank's step time on every rank
        assert value == pytest.approx(1.0e9 * 2 / 2.0e-3 / 1e9)  # both ranks' bytes over 2 ms
        assert printed == ""


def test_single_process_is_rank_zero_of_one(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    assert bench.world_info() == (1, 0, 0)
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
    assert bench.job_value(2.0e9, 1, 1.0) == pytest.approx(2000.0)
