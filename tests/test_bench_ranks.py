"""Multi-rank host logic of bench.py on CPU: two gloo ranks (the same code runs on
NCCL, one rank per GPU, under torchrun)."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        sync = bench.RankSync(world, None)
        sync.barrier()
        # each rank's timed region differs: the reported step time is the slowest rank's
        slowest = sync.max(4.0 + rank)
        sync.barrier()
        q.put((rank, slowest, bench.job_tokens_per_s(slowest, world)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_scale_weakly():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, tok_s in got:
        assert slowest == 5.0
        # weak scaling: every rank processes its own 16384 tokens per step
        assert abs(tok_s - 2 * 16384 / 5e-3) < 1e-6 * tok_s


def test_reference_arm_only_rank0_prints(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert buf.getvalue() == ""


def test_reference_arm_line_on_rank0(monkeypatch):
    """The oracle arm's JSON line carries the contract's keys, its own cpu_baseline and a
    zero-copy e2e, with value = the sample's tokens / the measured step time."""
    import json

    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert abs(line["value"] - bench.SAMPLE_TOKENS / (line["ms_per_step"] * 1e-3)) <= 0.01 * line["value"]
