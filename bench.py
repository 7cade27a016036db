#!/usr/bin/env python
"""Benchmark: one CSA prefill layer (T = 32768, 64 heads x dim 128, MQA KV dim 128,
4:1 overlapping compression -> 8192 entries, NVFP4 indexer 4 x 64, top-k 512,
raw window 128, sink) per step, on synthetic seeded inputs.

One JSON line on rank 0:
  value      tokens/s of the whole job (inputs resident in HBM), max over ranks
  e2e        the same through the C ABI with host buffers: pinned H2D of every
             input, the layer, D2H of the output, all inside the timed region;
             step i's upload and step i-1's download overlap step i's
             neighbours' compute (separate streams, two buffer sets)
  roofline   the dominant kernel (sparse_attn_fwd, tensor-bound): algorithmic
             FLOPs per launch / its CUDA-event duration inside the timed region,
             against the measured bf16 peak
  kernels    per-kernel average duration (ms) and algorithmic rate
  cpu_baseline  the CPU oracle on a bounded sample of the same workload

The default run also measures the two other throughputs the metric names and
reports them under "workloads" in the same line, each with its own roofline,
e2e, clocks and CPU baseline:
  csa_decode_32x1m    decode steps/s: 32 sequences x 1,048,576 cached tokens,
                      128 heads, top-k 1024, one new token per sequence per
                      step, replayed from a CUDA graph
  hca_prefill_2x128k  HCA prefill tokens/s: B = 2, T = 131072, 64 heads,
                      ratio 128 (1024 entries per sequence), window + sink
Each is also a line of its own with --workload.

--impl reference times the CPU oracle as the reference arm (rank 0 only).
Multi-GPU (torchrun): every rank runs its own independent layer (weak scaling,
no collective on the data path; the timing uses a MAX all-reduce).
"""
from __future__ import annotations

import argparse
import contextlib
import datetime
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA attn-layer prefill tokens/s & 1M-ctx decode steps/s; % of roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--chunk", type=int, default=0, help="query rows per indexer/top-k chunk (0 = all)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=4096, help="query rows in the CPU-oracle sample (about 10 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=0,
                    help="profiling case: override the layer's token count (not a bench line)")
    ap.add_argument("--workload", default="csa_prefill_32k",
                    choices=["csa_prefill_32k", "csa_decode_32x1m", "hca_prefill_2x128k", "stack_hhcc_256k",
                             "grouped_out_proj_32k"],
                    help="csa_prefill_32k (the default line), csa_decode_32x1m (decode steps/s), "
                         "hca_prefill_2x128k (HCA prefill tokens/s) or stack_hhcc_256k (4-layer prefill stack)")
    ap.add_argument("--no-extra", action="store_true",
                    help="default run only: skip the decode and HCA measurements under 'workloads'")
    ap.add_argument("--fused", action="store_true",
                    help="CSA prefill: score and select in the fused indexer_topk kernel")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def algorithmic_work(cfg):
    """Per-layer algorithmic work of each step (definitions in the design notes)."""
    T, H, D, m, k, W, S = cfg.T, cfg.H, cfg.D, cfg.m, cfg.k, cfg.W, cfg.S
    HI, DI = cfg.HI, cfg.DI
    rows = sel = vis_pairs = 0
    for t in range(T):
        vis = min(S, (t + 1) // m)
        vis_pairs += vis
        sel += min(k, vis) + min(W, t + 1)
    B = cfg.B
    esz = 2
    return {
        "attn_flops": B * 4.0 * H * D * sel,
        "attn_rows": B * sel,
        "indexer_pairs": B * vis_pairs,
        "indexer_flops": B * 2.0 * vis_pairs * HI * DI,
        "indexer_bytes": B * (vis_pairs * esz + T * HI * (DI // 2 + DI // 16 + 4) + S * (DI // 2 + DI // 16)),
        "topk_bytes": B * (vis_pairs * esz + T * k * 4),
        # fused indexer -> top-k: its inputs once and the indices; no score bytes
        "indexer_topk_bytes": B * (T * HI * (DI // 2 + DI // 16 + 4) + S * (DI // 2 + DI // 16) + T * k * 4),
        "compress_bytes": B * (3 * T * D * esz + S * D * esz),
        "compress_keys_bytes": B * (3 * T * DI * esz + S * (DI // 2 + DI // 16)),
        "quant_bytes": B * (T * HI * DI * esz + T * HI * (DI // 2 + DI // 16)),
        "attn_hbm_bytes": B * (2 * T * H * D * esz + T * k * 4),
    }


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.4)

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        samples = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    samples.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [s for s in samples if t0 - 0.05 <= s[0] <= t1 + 0.05] or samples[-3:]
        if not inside:
            return None
        mhz = sorted(s[1] for s in inside)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for s in inside for i, v in enumerate(s[3]) if v.lower().startswith("active")})
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": max(s[2] for s in inside), "reasons": reasons,
                "samples": len(inside)}


class OracleSample:
    """The CPU oracle as it stands, timed on a bounded sample of the layer:
    the compressors + NVFP4 quantisation once over all T tokens, then
    indexer/top-k/attention on batches of query rows (uniform, seed 1234);
    throughput = T / (t_compress + t_per_row * T)."""

    def __init__(self, cfg):
        import numpy as np
        import oracle
        from long_context_compressed_compress_b200 import inputs
        self.np, self.oracle, self.cfg = np, oracle, cfg
        # host inputs converted to float64 once (the oracle's working precision);
        # q stays in its storage dtype and the oracle converts the rows it reads
        self.x = {k: (v if k == "q" else v.to(torch_f64()).numpy())
                  for k, v in inputs.layer_inputs(cfg, device="cpu").items()}
        self.pos = np.arange(cfg.T)[None]
        self.rng = np.random.default_rng(1234)
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:  # pragma: no cover
            self.cores = 1
        c, x = cfg, self.x
        t0 = time.perf_counter()
        self.kv = oracle.round_out(oracle.csa_compress(x["a"], x["b"], x["z"], c.m), c.dtype)
        ks = oracle.round_out(oracle.csa_compress(x["a_I"], x["b_I"], x["z_I"], c.m), c.dtype)
        self.khat = oracle.nvfp4_quantize(ks)["xhat"]
        self.t_comp = time.perf_counter() - t0
        self.t_rows = 0.0
        self.n_rows = 0

    def rows(self, n):
        np, o, c, x = self.np, self.oracle, self.cfg, self.x
        ts = self.rng.integers(0, c.T, size=n)
        t0 = time.perf_counter()
        for t in ts:
            t = int(t)
            pos = np.array([[t]])
            qhat = o.nvfp4_quantize(x["q_I"][:, t:t + 1])["xhat"]
            sc = o.round_scores(o.indexer_score(qhat, self.khat, x["w"][:, t:t + 1], pos, c.m),
                                "bf16" if c.dtype != "f32" else "f32")
            idx = o.topk_select(sc, pos, c.m, c.k)
            o.sparse_attn(x["q"], self.kv, {(0, t): idx[0, 0]}, x["kv_raw"], c.T, x["sink"], c.tau, c.W, self.pos,
                          rows=[(0, t)])
        dt = time.perf_counter() - t0
        self.t_rows += dt
        self.n_rows += n
        return dt

    def value(self):
        per_row = self.t_rows / max(1, self.n_rows)
        return self.cfg.B * self.cfg.T / (self.t_comp + per_row * self.cfg.B * self.cfg.T)

    def single_thread(self, n_rows):
        """The same sample on one host thread (numpy's pools limited to 1):
        compressors again, then ``n_rows`` query rows; tokens/s."""
        try:
            from threadpoolctl import threadpool_limits
        except ImportError:  # pragma: no cover
            return None
        o, c, x = self.oracle, self.cfg, self.x
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            o.csa_compress(x["a"], x["b"], x["z"], c.m)
            o.nvfp4_quantize(o.round_out(o.csa_compress(x["a_I"], x["b_I"], x["z_I"], c.m), c.dtype))
            t_comp = time.perf_counter() - t0
            keep = (self.t_rows, self.n_rows)
            self.t_rows, self.n_rows = 0.0, 0
            self.rows(n_rows)
            per_row = self.t_rows / max(1, self.n_rows)
            self.t_rows, self.n_rows = keep
        return c.B * c.T / (t_comp + per_row * c.B * c.T)

    def describe(self, one_thread=None):
        d = {"value": self.value(), "unit": "tokens/s", "cores": self.cores, "kind": "oracle",
             "sample": f"compressors + NVFP4 over all {self.cfg.T} tokens ({self.t_comp:.1f} s), then "
                       f"indexer/top-k/attention on {self.n_rows} uniform query rows "
                       f"({self.t_rows:.1f} s), extrapolated to {self.cfg.T} rows"}
        if one_thread is not None:
            d["value_1thread"] = one_thread
        return d


def torch_f64():
    import torch
    return torch.float64


def cpu_baseline(cfg, n_rows):
    s = OracleSample(cfg)
    s.rows(n_rows)
    return s.describe(one_thread=s.single_thread(max(64, n_rows // 16)))


def run_reference(args, cfg, rank):
    """Reference arm: the CPU oracle, each step a bounded sample of query rows."""
    if rank != 0:
        return
    per_step = 64          # query rows of oracle work per step (about 0.1 s)
    s = OracleSample(cfg)
    for _ in range(args.warmup):
        s.rows(1)
    s.t_rows, s.n_rows = 0.0, 0
    for _ in range(args.steps):
        s.rows(per_step)
    v = s.value()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": cfg.B * cfg.T / v * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) inputs, U(0,1) indexer weights, N(0,1) sink)",
        "config": {"workload": "csa_prefill_32k" if not args.T else f"csa_prefill_T{cfg.T}", "B": cfg.B, "T": cfg.T, "H": cfg.H, "D": cfg.D, "m": cfg.m,
                   "S": cfg.S, "k": cfg.k, "HI": cfg.HI, "DI": cfg.DI, "W": cfg.W},
        "cpu_baseline": s.describe(),
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(ms, device):
    """The slowest rank's device time: every rank runs the same collective."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms):
    """Whole-job tokens/s: every rank processes its own replica of the workload."""
    return world * tokens_per_rank / (ms * 1e-3)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from long_context_compressed_compress_b200 import configs
    cfg = configs.CSA_PREFILL
    if args.T:
        cfg = configs.scaled(cfg, T=args.T)
    if args.workload == "csa_decode_32x1m":
        main_decode(args, rank, world, local)
        return
    if args.workload == "hca_prefill_2x128k":
        main_hca(args, rank, world, local)
        return
    if args.workload == "stack_hhcc_256k":
        main_stack(args, rank, world, local)
        return
    if args.workload == "grouped_out_proj_32k":
        main_outproj(args, rank, world, local)
        return
    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import inputs, layer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    peaks = load_peaks()
    work = algorithmic_work(cfg)
    x = inputs.layer_inputs(cfg, device="cuda")
    lay = layer.CsaPrefill(cfg, chunk=args.chunk or None, fused=args.fused)
    stream = torch.cuda.current_stream()

    # per-kernel CUDA events on the launching stream, inside the timed region
    ev = {}

    @contextlib.contextmanager
    def timer(name):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        yield
        e1.record(stream)
        ev.setdefault(name, []).append((e0, e1))

    for _ in range(args.warmup):
        lay.run(x)
    torch.cuda.synchronize()
    ev.clear()

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid) if hasattr(
        torch.cuda.get_device_properties(dev), "uuid") else str(local)
    sampler = ClockSampler(gpu_uuid)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        lay.run(x, timer=timer)
    s1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    ms_total = s0.elapsed_time(s1)
    if world > 1:
        ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    kern = {}
    for name, lst in ev.items():
        kern[name] = sum(a.elapsed_time(b) for a, b in lst) / args.steps
    launches = lay.launches * args.steps

    # ---- end to end through the C ABI with host buffers (copies overlapped across steps)
    host = {k: v.to("cpu").pin_memory() for k, v in x.items()}
    outs_host = [torch.empty(lay.out.shape, dtype=lay.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    e2e_ms = float("nan")
    if args.e2e_steps > 0:
        lays = [lay, layer.CsaPrefill(cfg, chunk=args.chunk or None, fused=args.fused)]
        xds = [{k: torch.empty_like(v) for k, v in x.items()} for _ in range(2)]
        e2e_ms = pipelined_e2e(lays, host, xds, outs_host, args.e2e_steps, world)
        barrier()
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, dev)
        del lays, xds
        torch.cuda.empty_cache()

    tokens = cfg.B * cfg.T
    value = job_throughput(world, tokens, ms_step)
    attn_ms = kern.get("sparse_attn_fwd", float("nan"))
    achieved = work["attn_flops"] / (attn_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = None
    # DRAM bytes per launch from the committed ncu summary, used only while the
    # attention sources still hash to what was profiled
    prof = os.path.join(ROOT, "profiles", "sparse_attn_fwd_csa_prefill_32k.md")
    if os.path.exists(prof) and not args.T:
        fields = {}
        with open(prof) as f:
            for ln in f:
                if ":" in ln and ln.split(":")[0] in ("kernel_hash", "dram_bytes_per_launch"):
                    fields[ln.split(":")[0]] = ln.split(":", 1)[1].strip()
        if fields.get("kernel_hash") == kernel_hash():
            traffic = int(fields["dram_bytes_per_launch"])
    rates = {
        "csa_compress": ("GB/s", work["compress_bytes"]),
        "csa_compress_indexer_keys": ("GB/s", work["compress_keys_bytes"]),
        "nvfp4_quantize": ("GB/s", work["quant_bytes"]),
        "indexer_score": ("GB/s", work["indexer_bytes"]),
        "topk_select": ("GB/s", work["topk_bytes"]),
        "indexer_topk": ("GB/s", work["indexer_topk_bytes"]),
        "sparse_attn_fwd": ("TFLOP/s", work["attn_flops"]),
    }
    kernels = {}
    for name, t in kern.items():
        unit, amount = rates.get(name, ("", 0))
        rate = amount / (t * 1e-3) / (1e9 if unit == "GB/s" else 1e12) if t > 0 else None
        pk = peaks["hbm_gbs"] if unit == "GB/s" else peak
        kernels[name] = {"ms": round(t, 5), "achieved": rate and round(rate, 2), "unit": unit,
                         "frac": rate and round(rate / pk, 4)}
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs, U(0,1) indexer weights, N(0,1) sink)",
        "config": {"workload": "csa_prefill_32k", "B": cfg.B, "T": cfg.T, "H": cfg.H, "D": cfg.D, "m": cfg.m,
                   "S": cfg.S, "k": cfg.k, "HI": cfg.HI, "DI": cfg.DI, "W": cfg.W,
                   "chunk": lay.chunk, "indexer_topk": "fused" if lay.fused else "two kernels",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (q + out = 1.07 GB per step)"},
        # no end-to-end number when no e2e step was timed (--e2e-steps 0)
        "e2e": {"value": job_throughput(world, tokens, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                "copies": "overlapped across steps (upload, compute, download streams)"} if args.e2e_steps > 0 else None,
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "kernel": "sparse_attn_fwd", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": work["attn_flops"]},
        "kernels": kernels,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_rows)
    if not args.no_extra and not args.T:
        # the metric's other two throughputs, measured in the same run (every
        # rank runs them, in the same order, as independent replicas)
        del x, host, outs_host, lay
        torch.cuda.empty_cache()
        extra = {}
        for name, fn in (("csa_decode_32x1m", measure_decode), ("hca_prefill_2x128k", measure_hca)):
            sub = fn(args, rank, world, dev)
            torch.cuda.empty_cache()
            extra[name] = {k: sub[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup", "config",
                                               "roofline", "kernels", "e2e", "gpu_launches", "clocks",
                                               "cpu_baseline") if k in sub}
        extra["variants"] = measure_variants(args, rank, world, dev)
        extra["kv_state"] = measure_state(args, rank, world, dev)
        extra["grouped_out_proj"] = measure_outproj(args, rank, world, dev)
        extra["indexer_topk"] = measure_fused_topk(args, rank, world, dev)
        line["workloads"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def decode_cpu_baseline(cfg, n_seq=2):
    """The oracle's decode step on ``n_seq`` sequences of the same cache recipe
    (state converted to float64 beforehand, not timed), extrapolated to B."""
    import numpy as np
    import oracle
    from long_context_compressed_compress_b200 import inputs
    import torch
    st = inputs.decode_state(cfg)
    seqs = list(range(n_seq))
    f = lambda t: t.to(torch.float64).numpy()
    o = {"kv_c": f(st["kv_c"][seqs, :cfg.S0]), "khat": oracle.nvfp4_quantize(f(st["k_I_src"][seqs, :cfg.S0]))["xhat"],
         "ring": f(st["ring"][seqs]).copy()}
    slot0 = ((cfg.T0 // cfg.m - 1) % 2) * cfg.m
    for n in ("a", "b", "z", "a_I", "b_I", "z_I"):
        src = f(st["carry_" + n][seqs])
        buf = np.zeros((n_seq, 2 * cfg.m, src.shape[-1]))
        buf[:, slot0:slot0 + cfg.m] = src
        o["carry_" + n] = buf
    x = {k: f(v[seqs]) for k, v in inputs.decode_step_inputs(cfg, 0).items()}
    x["sink"] = f(st["sink"])
    t0 = time.perf_counter()
    oracle.csa_decode_step(o, x, cfg.T0, cfg.m, cfg.k, cfg.W, cfg.tau, cfg.dtype)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = 1
    d = {"value": 1.0 / (dt * cfg.B / n_seq), "unit": "steps/s", "cores": cores, "kind": "oracle",
         "sample": f"one decode step for {n_seq} of the {cfg.B} sequences ({dt:.1f} s), "
                   f"extrapolated to all {cfg.B}"}
    try:
        from threadpoolctl import threadpool_limits
        o1 = {k: (v[:1].copy() if isinstance(v, np.ndarray) and v.ndim >= 2 else v) for k, v in o.items()}
        x1 = {k: (v[:1] if k != "sink" else v) for k, v in x.items()}
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle.csa_decode_step(o1, x1, cfg.T0, cfg.m, cfg.k, cfg.W, cfg.tau, cfg.dtype)
            d["value_1thread"] = 1.0 / ((time.perf_counter() - t0) * cfg.B)
    except ImportError:  # pragma: no cover
        pass
    return d


def main_decode(args, rank, world, local):
    """CSA decode at 1M context as a line of its own (see ``measure_decode``)."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import build, configs
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.impl == "reference":
        if rank == 0:
            cfg = configs.CSA_DECODE
            cb = decode_cpu_baseline(cfg)
            print(json.dumps({"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "steps/s",
                              "n_gpus": args.gpus, "steps": 1, "warmup": 0, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                              "config": {"workload": "csa_decode_32x1m"}, "cpu_baseline": cb,
                              "e2e": {"value": cb["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    line = measure_decode(args, rank, world, dev)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_decode(args, rank, world, dev):
    """CSA decode at 1M context: B = 32 sequences x 1,048,576 cached tokens
    (262,144 entries), H = 128, k = 1024; one step = one new token for every
    sequence, replayed from a CUDA graph.  value = steps/s of the whole job.
    At least 64 steps are timed (a multiple of m = 4, so entry emission is
    amortised as in the workload's definition)."""
    import dataclasses
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import configs, inputs, layer
    steps = max(64, args.steps)
    n_kern = 8
    total = args.warmup + steps + 2 * (args.e2e_steps + 2) + n_kern + 8
    cfg = dataclasses.replace(configs.CSA_DECODE, steps=total)
    peaks = load_peaks()
    st = inputs.decode_state(cfg, device="cuda")
    lay = layer.CsaDecode(cfg, st, cfg.T0)
    stream = torch.cuda.current_stream()
    x = inputs.decode_step_inputs(cfg, 0, device="cuda")
    # per-kernel breakdown: eager steps with events around each call
    ev = {}

    @contextlib.contextmanager
    def timer(name):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        yield
        e1.record(stream)
        ev.setdefault(name, []).append((e0, e1))

    lay.step(x)
    torch.cuda.synchronize()
    for _ in range(n_kern):
        lay.step(x, timer=timer)
    torch.cuda.synchronize()
    kern = {k: sum(a.elapsed_time(b) for a, b in v) / n_kern for k, v in ev.items()}
    lay.capture(x)
    for _ in range(args.warmup):
        lay.replay()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(dev.index))
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(steps):
        lay.replay()
    s1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    ms = s0.elapsed_time(s1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    ms_step = ms / steps
    # end to end: pinned host inputs copied in, the graph, the output read back
    host = {k: v.cpu().pin_memory() for k, v in x.items()}
    out_host = torch.empty(lay.out.shape, dtype=lay.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        for k, v in host.items():
            lay.x[k].copy_(v, non_blocking=True)
        lay.replay()
        out_host.copy_(lay.out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / max(1, args.e2e_steps)
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dev)
    # roofline of the dominant kernel (the indexer: reads every visible NVFP4 key)
    B, DI, HI = cfg.B, cfg.DI, cfg.HI
    n_vis = (cfg.T0 + 1) // cfg.m
    idx_bytes = B * (n_vis * (DI // 2 + DI // 16) + n_vis * 2 + HI * (DI // 2 + DI // 16 + 4))
    topk_bytes = B * (n_vis * 2 + cfg.k * 4)
    attn_bytes = B * (cfg.H * cfg.D * 2 * 2 + (cfg.k + cfg.W) * cfg.D * 2 + cfg.k * 4)
    rates = {"indexer_score": idx_bytes, "topk_select": topk_bytes, "sparse_attn_fwd": attn_bytes}
    kernels = {}
    for name, t in kern.items():
        amount = rates.get(name)
        rate = amount / (t * 1e-3) / 1e9 if amount and t > 0 else None
        kernels[name] = {"ms": round(t, 5), "achieved": rate and round(rate, 1), "unit": "GB/s" if rate else "",
                         "frac": rate and round(rate / peaks["hbm_gbs"], 4)}
    it = kern["indexer_score"]
    achieved = idx_bytes / (it * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": world / (ms_step * 1e-3), "unit": "steps/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic cache drawn on the device (N(0,1) entries and indexer keys, seeded)",
        "config": {"workload": "csa_decode_32x1m", "B": B, "T0": cfg.T0, "S0": cfg.S0, "H": cfg.H, "D": cfg.D,
                   "HI": HI, "DI": DI, "k": cfg.k, "W": cfg.W, "graph": True,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (302 MB of NVFP4 keys and 2.1 GB of KV per step's cache)"},
        "e2e": {"value": job_throughput(world, 1, e2e_ms), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms} if args.e2e_steps > 0 else None,
        "gpu_launches": lay.launches * steps,
        "roofline": {"bound": "hbm", "kernel": "indexer_score", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peaks['source']} hbm_gbs", "algorithmic_bytes_per_launch": idx_bytes},
        "kernels": kernels, "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = decode_cpu_baseline(configs.CSA_DECODE)
    lay.graph = None
    return line


def hca_cpu_baseline(cfg, x, n_rows=64, one_thread=True):
    """The oracle's HCA layer on the host cores: the 128:1 compression of every
    token, then dense attention for ``n_rows`` uniform query rows (seed 1234),
    extrapolated to all B*T rows; the inputs are the device draw copied to the
    host (outside the timed part), q only for the sampled rows."""
    import numpy as np
    import oracle
    import torch

    def run(rows_per_seq):
        rng = np.random.default_rng(1234)
        f = lambda t: t.to("cpu", torch.float64).numpy()
        host = [(f(x["a"][b]), f(x["z"][b]), f(x["kv_raw"][b])) for b in range(cfg.B)]
        ts = [np.sort(rng.integers(0, cfg.T, size=rows_per_seq)) for _ in range(cfg.B)]
        qs = [f(x["q"][b, torch.from_numpy(t).to(x["q"].device)]) for b, t in enumerate(ts)]
        sink = f(x["sink"])
        t0 = time.perf_counter()
        kvs = [oracle.round_out(oracle.hca_compress(a, z, cfg.m), cfg.dtype) for (a, z, _) in host]
        t_comp = time.perf_counter() - t0
        t0 = time.perf_counter()
        for b in range(cfg.B):
            n = len(ts[b])
            oracle.dense_attn(qs[b][None], kvs[b][None], host[b][2][None], cfg.T, sink, cfg.tau, cfg.W,
                              ts[b][None], cfg.m, rows=[(0, i) for i in range(n)])
        t_rows = time.perf_counter() - t0
        n_tot = cfg.B * rows_per_seq
        return cfg.B * cfg.T / (t_comp + t_rows / n_tot * cfg.B * cfg.T), t_comp, t_rows, n_tot

    v, t_comp, t_rows, n_tot = run(max(1, n_rows // cfg.B))
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        threadpool_limits, cores = None, 1
    d = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
         "sample": f"128:1 compression of all {cfg.B}x{cfg.T} tokens ({t_comp:.1f} s), then dense attention "
                   f"for {n_tot} uniform query rows ({t_rows:.1f} s), extrapolated to {cfg.B * cfg.T} rows"}
    if one_thread and threadpool_limits is not None:
        with threadpool_limits(limits=1):
            d["value_1thread"] = run(max(1, n_rows // (4 * cfg.B)))[0]
    return d


def main_hca(args, rank, world, local):
    """HCA prefill as a line of its own (see ``measure_hca``)."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import build, configs, inputs
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.impl == "reference":
        if rank == 0:
            cfg = configs.HCA_PREFILL
            x = inputs.layer_inputs(cfg, device="cuda")
            cb = hca_cpu_baseline(cfg, x, one_thread=False)
            print(json.dumps({"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
                              "n_gpus": args.gpus, "steps": 1, "warmup": 0, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                              "config": {"workload": "hca_prefill_2x128k"}, "cpu_baseline": cb,
                              "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    line = measure_hca(args, rank, world, dev)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_hca(args, rank, world, dev):
    """HCA prefill: B = 2, T = 131072, 64 heads x dim 128, ratio 128 (1024
    entries per sequence), window 128 + sink, gate logits N(0, 2); one step =
    hca_compress + hca_dense_attn_fwd on inputs resident in HBM.  value = B*T
    tokens per step time, whole job."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import configs, inputs, layer
    cfg = configs.HCA_PREFILL
    peaks = load_peaks()
    x = inputs.layer_inputs(cfg, device="cuda")
    lay = layer.HcaPrefill(cfg)
    stream = torch.cuda.current_stream()
    ev = {}

    @contextlib.contextmanager
    def timer(name):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        yield
        e1.record(stream)
        ev.setdefault(name, []).append((e0, e1))

    steps = max(3, min(args.steps, 40))
    for _ in range(args.warmup):
        lay.run(x)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(dev.index))
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(steps):
        lay.run(x, timer=timer)
    s1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    ms = s0.elapsed_time(s1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    ms_step = ms / steps
    kern = {k: sum(a.elapsed_time(b) for a, b in v) / steps for k, v in ev.items()}
    flops = attn_flops(cfg)
    comp_bytes = cfg.B * (2 * cfg.T * cfg.D * 2 + cfg.S * cfg.D * 2)
    kernels = {}
    for name, t in kern.items():
        if name == "hca_dense_attn_fwd":
            rate = flops / (t * 1e-3) / 1e12
            kernels[name] = {"ms": round(t, 4), "achieved": round(rate, 1), "unit": "TFLOP/s",
                             "frac": round(rate / peaks["bf16_tflops"], 4)}
        else:
            rate = comp_bytes / (t * 1e-3) / 1e9
            kernels[name] = {"ms": round(t, 4), "achieved": round(rate, 1), "unit": "GB/s",
                             "frac": round(rate / peaks["hbm_gbs"], 4)}
    achieved = flops / (kern["hca_dense_attn_fwd"] * 1e-3) / 1e12
    # end to end: pinned host inputs in, the layer, the output back
    n_e2e = max(2, min(args.e2e_steps, 4)) if args.e2e_steps > 0 else 0
    e2e = None
    if n_e2e:
        host = {k: v.cpu().pin_memory() for k, v in x.items()}
        outs_host = [torch.empty(lay.out.shape, dtype=lay.out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = outs_host[0].numel() * outs_host[0].element_size()
        lays = [lay, layer.HcaPrefill(cfg)]
        xds = [x, {k: torch.empty_like(v) for k, v in x.items()}]
        e2e_ms = pipelined_e2e(lays, host, xds, outs_host, n_e2e, world)
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, dev)
        e2e = {"value": job_throughput(world, cfg.B * cfg.T, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": n_e2e, "copies": "overlapped across steps (upload, compute, download streams)"}
        del host, outs_host, lays, xds
        torch.cuda.empty_cache()
    line = {
        "metric": METRIC, "value": job_throughput(world, cfg.B * cfg.T, ms_step), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded inputs drawn on the device: a N(0,1), z N(0,2), q, kv_raw, sink N(0,1))",
        "config": {"workload": "hca_prefill_2x128k", "B": cfg.B, "T": cfg.T, "H": cfg.H, "D": cfg.D, "m": cfg.m,
                   "S": cfg.S, "W": cfg.W, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (q + out = 8.6 GB per step)"},
        "e2e": e2e,
        "gpu_launches": lay.launches * steps,
        "roofline": {"bound": "tensor", "kernel": "hca_dense_attn_fwd", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": None, "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": flops},
        "kernels": kernels, "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = hca_cpu_baseline(cfg, x)
    del x, lay
    return line


def measure_variants(args, rank, world, dev):
    """The same kernels at the variant settings the pages name: top-k 32 / 512
    / 1024 on the CSA prefill workload and HCA ratio 64 on the HCA prefill
    workload.  A short timed run each (inputs resident, per-kernel events);
    tokens/s and the attention kernel's fraction of the bf16 burst peak."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import configs, inputs, layer
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    res = {}
    cases = [("csa_prefill_32k_k32", configs.CSA_PREFILL_K32), ("csa_prefill_32k", configs.CSA_PREFILL),
             ("csa_prefill_32k_k1024", configs.CSA_PREFILL_K1024),
             ("hca_prefill_2x128k_ratio64", configs.HCA_PREFILL_M64)]
    for name, cfg in cases:
        x = inputs.layer_inputs(cfg, device="cuda")
        lay = layer.CsaPrefill(cfg) if cfg.kind == "csa" else layer.HcaPrefill(cfg)
        attn = "sparse_attn_fwd" if cfg.kind == "csa" else "hca_dense_attn_fwd"
        ev = {}

        @contextlib.contextmanager
        def timer(nm):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            yield
            e1.record(stream)
            ev.setdefault(nm, []).append((e0, e1))

        steps = 10 if cfg.kind == "csa" else 4
        for _ in range(3):
            lay.run(x)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(steps):
            lay.run(x, timer=timer)
        s1.record(stream)
        torch.cuda.synchronize()
        ms = s0.elapsed_time(s1)
        if world > 1:
            ms = max_over_ranks(ms, dev)
        kern = {k: sum(a.elapsed_time(b) for a, b in v) / steps for k, v in ev.items()}
        fl = attn_flops(cfg)
        tf = fl / (kern[attn] * 1e-3) / 1e12
        res[name] = {"k" if cfg.kind == "csa" else "m": cfg.k if cfg.kind == "csa" else cfg.m,
                     "value": job_throughput(world, cfg.B * cfg.T, ms / steps), "unit": "tokens/s",
                     "ms_per_step": ms / steps, "steps": steps,
                     "attention": {"kernel": attn, "ms": round(kern[attn], 4), "achieved": round(tf, 1),
                                   "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4)},
                     "kernels_ms": {k: round(v, 4) for k, v in kern.items()}}
        del x, lay
        torch.cuda.empty_cache()
    return res


def measure_state(args, rank, world, dev):
    """KV-cache state management on the CSA prefill workload: the every-1024
    snapshots of the raw window and compressor carries (one launch per tensor,
    32 snapshots of B = 1, T = 32768) and one restore into a decode state.
    Algorithmic bytes: each snapshot slot read once and written once."""
    import dataclasses
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import configs, inputs, layer
    cfg = configs.CSA_PREFILL
    peaks = load_peaks()
    x = inputs.layer_inputs(cfg, device="cuda")
    pre = layer.CsaPrefill(cfg)
    pre.run(x)
    stream = torch.cuda.current_stream()
    reps = 20
    for _ in range(3):
        ck = layer.PrefixCheckpoints(cfg, x)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        ck = layer.PrefixCheckpoints(cfg, x)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    n = len(ck.positions)
    bytes_ = 2 * 2 * cfg.B * n * (cfg.W * cfg.D + 2 * cfg.m * (3 * cfg.D + 3 * cfg.DI))
    dcfg = dataclasses.replace(configs.CSA_DECODE, B=cfg.B, T0=ck.positions[-1] + 1, H=cfg.H, k=cfg.k, steps=4)
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    dec = ck.restore(dcfg, n - 1, pre.kv_c, pre.k_fp4, pre.k_sf, extra_entries=2)
    r1.record(stream)
    torch.cuda.synchronize()
    res = {"snapshots": n, "every": ck.every, "checkpoint_ms": round(ms, 5),
           "checkpoint_bytes": bytes_, "checkpoint_GBps": round(bytes_ / (ms * 1e-3) / 1e9, 1),
           "checkpoint_frac": round(bytes_ / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "restore_ms": round(r0.elapsed_time(r1), 4),
           "restored_cache_entries": int(dec.cap), "launches": ck.launches}
    del x, pre, ck, dec
    return res


def main_outproj(args, rank, world, local):
    """The grouped output projection as a line of its own (see ``measure_outproj``)."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import build
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "unavailable": "no CPU timing of a 3.3 TFLOP projection; "
                              "its oracle runs on sampled rows in the tests"}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    r = measure_outproj(args, rank, world, dev)
    line = {"metric": METRIC, "value": r["achieved"], "unit": "TFLOP/s", "n_gpus": world, "steps": r["reps"],
            "warmup": 3, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) activations, scaled N(0,1) weights)",
            "config": {"workload": "grouped_out_proj_32k", **{k: r[k] for k in ("M", "H", "D", "groups", "d_g",
                                                                                 "d_model")}},
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel", "achieved": r["achieved"], "peak": r["peak"],
                         "unit": "TFLOP/s", "frac": r["frac"], "traffic": None},
            "gpu_launches": r["launches"] * r["reps"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_outproj(args, rank, world, dev):
    """Grouped output projection after a 128-head attention layer: M = 32768
    rows, H = 128 x D = 128, 8 groups of 16 heads projected to 1024 each, then
    to a model dimension of 4096 (two tcgen05 GEMM launches; bf16 in, fp32
    accumulation).  Algorithmic FLOPs: 2 M (H D d_g + g d_g d_model)."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import ops
    peaks = load_peaks()
    M, H, D, g, d_g, d_model = 32768, 128, 128, 8, 1024, 4096
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9)
    o = torch.randn((M, H, D), generator=gen, device="cuda").to(torch.bfloat16)
    w1 = (torch.randn((g, d_g, H // g * D), generator=gen, device="cuda") / (H // g * D) ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((d_model, g * d_g), generator=gen, device="cuda") / (g * d_g) ** 0.5).to(torch.bfloat16)
    y = torch.empty((M, g * d_g), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((M, d_model), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(3):
        ops.grouped_out_proj(o, w1, w2, y, out)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    reps = max(2, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        ops.grouped_out_proj(o, w1, w2, y, out)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    flops = 2.0 * M * (H * D * d_g + g * d_g * d_model)
    plain = 2.0 * M * H * D * d_model
    tf = flops / (ms * 1e-3) / 1e12
    res = {"M": M, "H": H, "D": D, "groups": g, "d_g": d_g, "d_model": d_model, "ms": round(ms, 4),
           "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": peaks["bf16_tflops"],
           "frac": round(tf / peaks["bf16_tflops"], 4), "flops": flops,
           "flops_vs_ungrouped": round(flops / plain, 3), "launches": 2, "reps": reps}
    del o, w1, w2, y, out
    torch.cuda.empty_cache()
    return res


def pipelined_e2e(lays, host, xds, outs_host, steps, world):
    """End-to-end steps through the public API with host buffers, the copies
    overlapped across steps: step i uploads its inputs (pinned host -> buffer
    set i % 2) on an upload stream, runs the layer on the compute stream and
    downloads its output on a download stream, so step i's compute runs while
    step i + 1 uploads and step i - 1 downloads (PCIe is full duplex).  Every
    step still moves all of its input and output bytes.  Returns ms per step,
    from the first upload to the last download, after two warm-up steps."""
    import torch
    import torch.distributed as dist
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    out_free = [torch.cuda.Event(), torch.cuda.Event()]
    used = [False, False]

    def step(i):
        b = i & 1
        if used[b]:
            up.wait_event(done[b])          # step i - 2 has finished reading buffer set b
        with torch.cuda.stream(up):
            for k, v in host.items():
                xds[b][k].copy_(v, non_blocking=True)
        in_ready[b].record(up)
        comp.wait_event(in_ready[b])
        if used[b]:
            comp.wait_event(out_free[b])    # step i - 2's output has been downloaded
        lays[b].run(xds[b])
        done[b].record(comp)
        down.wait_event(done[b])
        with torch.cuda.stream(down):
            outs_host[b].copy_(lays[b].out, non_blocking=True)
        out_free[b].record(down)
        used[b] = True

    step(0)
    step(1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(steps):
        step(i)
    comp.wait_event(out_free[0])
    comp.wait_event(out_free[1])
    e1.record(comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def measure_fused_topk(args, rank, world, dev):
    """Indexer score + top-k on the CSA prefill shapes (T = 32768, S = 8192,
    k = 512): the fused kernel (scores kept on chip) against indexer_score +
    topk_select (BF16 scores through HBM), on the same NVFP4 inputs, with the
    two index tensors compared bit for bit."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import configs, inputs, layer, ops
    cfg = configs.CSA_PREFILL
    lay = layer.CsaPrefill(cfg, fused=False)
    x = inputs.layer_inputs(cfg, device="cuda")
    lay.run(x)
    torch.cuda.synchronize()
    idx_f = torch.empty_like(lay.idx)
    stream = torch.cuda.current_stream()

    def fused():
        ops.indexer_topk(lay.q_fp4, lay.q_sf, lay.k_fp4, lay.k_sf, x["w"], lay.q_pos0, idx_f, cfg.S, cfg.m)

    def unfused():
        ops.indexer_score(lay.q_fp4, lay.q_sf, lay.k_fp4, lay.k_sf, x["w"], lay.q_pos0, lay.score, cfg.S, cfg.m)
        ops.topk_select(lay.score, lay.idx, cfg.S, cfg.m, lay.q_pos0)

    res = {"config": "csa_prefill_32k (T 32768, S 8192, k 512, HI 4)"}
    reps = max(2, min(args.steps, 10))
    for name, fn in (("fused_ms", fused), ("unfused_ms", unfused)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = round(max_over_ranks(ms, dev) if world > 1 else ms, 4)
    res["bit_identical"] = bool(torch.equal(idx_f, lay.idx))
    res["launches"] = {"fused": 1, "unfused": 2}
    del lay, x, idx_f
    torch.cuda.empty_cache()
    return res


def attn_flops(cfg):
    """4·H·D flops per (query, head, attended row); rows = the selected (CSA) or
    all visible (HCA) entries plus the raw window, summed over queries."""
    import numpy as np
    t = np.arange(cfg.T, dtype=np.int64)
    vis = np.minimum(cfg.S, (t + 1) // cfg.m)
    ent = np.minimum(cfg.k, vis) if cfg.kind == "csa" else vis
    rows = int((ent + np.minimum(cfg.W, t + 1)).sum())
    return cfg.B * 4.0 * cfg.H * cfg.D * rows


def main_stack(args, rank, world, local):
    """Four prefill layers HCA, HCA, CSA, CSA at T = 262144, 128 heads x dim 128
    (CSA k = 1024, indexer 4 x 64; HCA ratio 128), independent seeded inputs per
    layer, all resident in HBM.  value = T / (time of the 4 layers) tokens/s."""
    import torch
    import torch.distributed as dist
    from long_context_compressed_compress_b200 import build, configs
    build.build()
    from long_context_compressed_compress_b200 import inputs, layer
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfgs = configs.STACK.layers
    if args.impl == "reference":
        if rank == 0:
            # the oracle on a row sample of each layer, extrapolated per layer
            tot = 0.0
            descr = []
            for c in cfgs:
                s = OracleSample(c) if c.kind == "csa" else None
                if s is None:
                    import numpy as np
                    import oracle
                    x = inputs.layer_inputs(c, device="cpu")
                    t0 = time.perf_counter()
                    oracle.hca_layer(x, c.m, c.W, c.tau, c.dtype, rows=[(0, int(r)) for r in
                                     np.random.default_rng(1234).integers(0, c.T, 4)])
                    dt = time.perf_counter() - t0
                    tot += dt / 4 * c.T
                    descr.append(f"HCA: 4 rows + compression {dt:.1f} s")
                else:
                    s.rows(4)
                    tot += c.T / s.value()
                    descr.append("CSA: " + s.describe()["sample"])
            v = cfgs[0].T / tot
            print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                              "n_gpus": args.gpus, "steps": 1, "warmup": 0, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                              "config": {"workload": "stack_hhcc_256k"},
                              "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(),
                                               "kind": "oracle", "sample": "; ".join(descr)},
                              "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks = load_peaks()
    xs = [inputs.layer_inputs(c, device="cuda") for c in cfgs]
    stk = layer.Stack(cfgs, chunk=args.chunk or 16384)
    stream = torch.cuda.current_stream()
    ev = {}

    @contextlib.contextmanager
    def timer(name):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        yield
        e1.record(stream)
        ev.setdefault(name, []).append((e0, e1))

    for _ in range(args.warmup):
        stk.run(xs)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(local))
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        stk.run(xs, timer=timer)
    s1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    ms = s0.elapsed_time(s1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    ms_step = ms / args.steps
    kern = {k: sum(a.elapsed_time(b) for a, b in v) / args.steps for k, v in ev.items()}
    flops = {"sparse_attn_fwd": sum(attn_flops(c) for c in cfgs if c.kind == "csa"),
             "hca_dense_attn_fwd": sum(attn_flops(c) for c in cfgs if c.kind == "hca")}
    kernels = {}
    for name, t in kern.items():
        f = flops.get(name)
        rate = f / (t * 1e-3) / 1e12 if f else None
        kernels[name] = {"ms": round(t, 4), "achieved": rate and round(rate, 1), "unit": "TFLOP/s" if f else "",
                         "frac": rate and round(rate / peaks["bf16_tflops_sustained"], 4)}
    top = max(flops, key=lambda n: kern.get(n, 0.0))
    achieved = flops[top] / (kern[top] * 1e-3) / 1e12
    # end to end: every layer's inputs copied from pinned host memory, the four
    # layers, the four outputs read back
    host = [{k: v.cpu().pin_memory() for k, v in x.items()} for x in xs]
    outs_h = [torch.empty(lay.out.shape, dtype=lay.out.dtype).pin_memory() for lay in stk.layers]
    h2d = sum(v.numel() * v.element_size() for h in host for v in h.values())
    d2h = sum(o.numel() * o.element_size() for o in outs_h)

    def e2e_step():
        for h, x in zip(host, xs):
            for k, v in h.items():
                x[k].copy_(v, non_blocking=True)
        stk.run(xs)
        for o, lay in zip(outs_h, stk.layers):
            o.copy_(lay.out, non_blocking=True)

    n_e2e = max(1, min(args.e2e_steps, 3))
    e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dev)
    T = cfgs[0].T
    line = {
        "metric": METRIC, "value": job_throughput(world, T, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs per layer, drawn on the device)",
        "config": {"workload": "stack_hhcc_256k", "layers": "HCA,HCA,CSA,CSA", "T": T, "H": cfgs[0].H,
                   "D": cfgs[0].D, "k": cfgs[2].k, "chunk": stk.layers[2].chunk,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (8.6 GB of q per layer)"},
        "e2e": {"value": job_throughput(world, T, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": stk.launches * args.steps,
        "roofline": {"bound": "tensor", "kernel": top, "achieved": achieved,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops_sustained"], "traffic": None,
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel inside a long step)",
                     "algorithmic_flops_per_step": flops[top]},
        "kernels": kernels, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def kernel_hash():
    import hashlib
    h = hashlib.sha1()
    for f in ("attn_tc.cu", "common.cuh", "attention.cu"):
        with open(os.path.join(ROOT, "long_context_compressed_compress_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


if __name__ == "__main__":
    main()
