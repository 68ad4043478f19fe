"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): the
max-over-ranks timing reduction, the whole-job throughput, and the reference
arm running on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r reports times r+1, 10-r: the reduction must return the per-slot max
    red = bench.max_over_ranks([float(rank + 1), float(10 - rank), 0.5 * rank], "cpu")
    ref_out = io.StringIO()
    with redirect_stdout(ref_out):
        rank_seen = bench.dist_setup()[1]
    q.put((rank, red, rank_seen))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, red, seen in out:
        assert red == [2.0, 10.0, 0.5]
        assert seen == rank


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1, 8192, 10, 1000.0) == 81920.0
    assert bench.job_throughput(4, 8192, 10, 1000.0) == 4 * 81920.0


def test_reference_arm_is_silent_off_rank0(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(bench.parse_args())
    assert buf.getvalue() == ""


def test_reference_arm_line_on_cpu(monkeypatch):
    """The reference arm (the CPU oracle) prints one contract line."""
    sys.path.insert(0, ROOT)
    import bench
    for v in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--config", "c0_tiny",
                                      "--steps", "2", "--warmup", "1"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(bench.parse_args())
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
