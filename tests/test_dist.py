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


# --------------------------------------------------- prefill split over ranks

def _shard_worker(rank, world, port, q, T):
    """One rank of a CPU (gloo) run of the prefill split's host side: the
    shard plan, the two halo exchanges and the entry all-gather, with the
    oracle's compressor standing in for the kernel on each shard."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from long_context_compressed_compress_b200 import configs, inputs, shard
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = configs.scaled(configs.PR1, T=T)
        x = inputs.layer_inputs(cfg, device="cpu")        # every rank draws the same full inputs
        plan = shard.ShardPlan(cfg.T, cfg.m, cfg.W, world)
        s, e = plan.rows(rank)
        xl = {k: (v if k == "sink" else v[:, s:e].contiguous()) for k, v in x.items()}
        # halos: the left neighbour's last block (compressor) and last W-1 raw rows
        pred = {n: shard.left_halo(xl[n], cfg.m) for n in ("a", "b", "z")}
        raw_halo = shard.left_halo(xl["kv_raw"], cfg.W - 1)
        ok_halo = all(torch.equal(pred[n], x[n][:, max(0, s - cfg.m):s]) for n in pred)
        h0, h1 = plan.raw_halo(rank)
        ok_halo = ok_halo and torch.equal(raw_halo, x["kv_raw"][:, h0:h1])
        # the ring the attention reads: every window token at slot j % raw_cap
        ring = shard.window_ring(raw_halo, xl["kv_raw"], s, cfg.W)
        ok_ring = all(torch.equal(ring[:, j % ring.shape[1]], x["kv_raw"][:, j]) for j in range(h0, e))
        # entries of the rank's own blocks (oracle compressor), gathered
        fhp = rank > 0
        src = [torch.cat([pred[n], xl[n]], dim=1) if fhp else xl[n] for n in ("a", "b", "z")]
        e_loc = torch.from_numpy(oracle.csa_compress(*src, m=cfg.m, first_has_pred=fhp))
        counts = [plan.entries(r)[1] - plan.entries(r)[0] for r in range(world)]
        full = shard.gather_entries(e_loc, counts).numpy()
        ref = oracle.csa_compress(x["a"], x["b"], x["z"], cfg.m)
        q.put((rank, ok_halo, ok_ring, full.shape == ref.shape and np.array_equal(full, ref), plan.start, plan.end))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 1024), (3, 1030)])
def test_prefill_split_exchange_gloo(world, T):
    """Shards cover the sequence in multiples of m; the compressor halo and
    the window halo are the left neighbour's rows; the window ring holds every
    row a shard's windows read; the all-gathered entries of the per-shard
    compressions equal the whole-sequence compression exactly."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q, T)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_halo, ok_ring, ok_entries, starts, ends in out:
        assert ok_halo and ok_ring and ok_entries, (rank, ok_halo, ok_ring, ok_entries)
        assert starts[0] == 0 and ends[-1] == T and all(s % 4 == 0 for s in starts)
        assert all(ends[i] == starts[i + 1] for i in range(world - 1))
