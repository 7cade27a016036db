"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the timing
reduction takes the slowest rank, and the job value counts every replica."""
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


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
        q.put((rank, ms, bench.job_throughput(world, 32768, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in out:
        assert ms == 2.5   # the slower rank's time, on every rank
        assert value == pytest.approx(2 * 32768 / 2.5e-3)


def test_reference_arm_is_rank0_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    from long_context_compressed_compress_b200 import configs

    class A:
        steps, warmup, gpus, T = 1, 0, 2, 0
    assert bench.run_reference(A(), configs.CSA_PREFILL, rank=1) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank0(capsys):
    """Rank 0 times the oracle on a bounded sample and prints one JSON line with
    the contract's keys (impl, metric/value/unit, cpu_baseline, zero-byte e2e)."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    from long_context_compressed_compress_b200 import configs

    class A:
        steps, warmup, gpus, T = 1, 0, 1, 512
    bench.run_reference(A(), configs.scaled(configs.CSA_PREFILL, T=512), rank=0)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["T"] == 512
