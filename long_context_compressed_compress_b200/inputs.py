"""Seeded synthetic inputs for the CSA/HCA workloads.

This module only draws random tensors in a fixed order; it contains none of the
layer's arithmetic.  Both the GPU library's tests/bench and the CPU oracle read
the tensors it returns.

Recipe: a ``torch.Generator`` on the target device seeded with the config's
seed; tensors are drawn in the order listed below as float32 N(0,1) (or U(0,1)
for the indexer weights w), multiplied by their stated scale, then rounded once
to the workload dtype.  Large tensors are drawn in row chunks of at most
``CHUNK`` elements so the float32 temporary stays small; the chunking is part of
the recipe.

CSA layer order: a, b, z, a_I, b_I, z_I, q_I, w, q, kv_raw, sink
HCA layer order: a, z, q, kv_raw, sink
"""
from __future__ import annotations

import torch

CHUNK = 1 << 26

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _draw(gen, shape, device, dtype, scale=1.0, kind="normal"):
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1) if out.numel() else out
    n = out.numel()
    row = 1
    for s in shape[1:]:
        row *= s
    step = max(row, (CHUNK // max(row, 1)) * max(row, 1))
    for off in range(0, n, step):
        cnt = min(step, n - off)
        if kind == "normal":
            x = torch.randn(cnt, generator=gen, device=device, dtype=torch.float32)
        else:
            x = torch.rand(cnt, generator=gen, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[off:off + cnt].copy_(x)
    return out


def layer_inputs(cfg, device="cpu", seed=None):
    """Inputs of one CSA or HCA layer (see module docstring for the order)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    dt = _DT[cfg.dtype]
    B, T, H, D = cfg.B, cfg.T, cfg.H, cfg.D
    x = {}
    if cfg.kind == "csa":
        x["a"] = _draw(gen, (B, T, D), device, dt)
        x["b"] = _draw(gen, (B, T, D), device, dt)
        x["z"] = _draw(gen, (B, T, D), device, dt, cfg.z_std)
        x["a_I"] = _draw(gen, (B, T, cfg.DI), device, dt)
        x["b_I"] = _draw(gen, (B, T, cfg.DI), device, dt)
        x["z_I"] = _draw(gen, (B, T, cfg.DI), device, dt)
        x["q_I"] = _draw(gen, (B, T, cfg.HI, cfg.DI), device, dt)
        x["w"] = _draw(gen, (B, T, cfg.HI), device, torch.float32, kind="uniform")
    else:
        x["a"] = _draw(gen, (B, T, D), device, dt)
        x["z"] = _draw(gen, (B, T, D), device, dt, cfg.z_std)
    x["q"] = _draw(gen, (B, T, H, D), device, dt, cfg.q_scale)
    x["kv_raw"] = _draw(gen, (B, T, D), device, dt)
    if cfg.sink == "zero":
        x["sink"] = torch.zeros(H, dtype=torch.float32, device=device)
    else:
        x["sink"] = _draw(gen, (H,), device, torch.float32)
    return x


def decode_state(cfg, device="cpu", extra_entries=None):
    """Synthetic decode cache at position T0 (the cache is drawn directly rather
    than produced by a 1M-token prefill): compressed KV entries, the indexer-key
    source values (quantised to NVFP4 by the caller), the raw-token ring of the
    last W tokens, and the raw (a,b,z,a_I,b_I,z_I) rows of the last complete
    block (the compressor carry).  Capacity leaves room for ``extra_entries``
    entries emitted during decoding.

    Order: kv_c, k_I_src, ring, carry a, b, z, a_I, b_I, z_I, sink [H].
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    dt = _DT[cfg.dtype]
    extra = cfg.steps // cfg.m + 1 if extra_entries is None else extra_entries
    cap = cfg.S0 + extra
    B, D, DI, m = cfg.B, cfg.D, cfg.DI, cfg.m
    st = {}
    st["kv_c"] = torch.zeros((B, cap, D), dtype=dt, device=device)
    st["kv_c"][:, : cfg.S0] = _draw(gen, (B, cfg.S0, D), device, dt)
    st["k_I_src"] = torch.zeros((B, cap, DI), dtype=dt, device=device)
    st["k_I_src"][:, : cfg.S0] = _draw(gen, (B, cfg.S0, DI), device, dt)
    st["ring"] = _draw(gen, (B, cfg.W, D), device, dt)
    for name, dim in (("a", D), ("b", D), ("z", D), ("a_I", DI), ("b_I", DI), ("z_I", DI)):
        st["carry_" + name] = _draw(gen, (B, m, dim), device, dt)
    st["sink"] = _draw(gen, (cfg.H,), device, torch.float32)
    return st


def decode_step_inputs(cfg, step, device="cpu"):
    """Per-step inputs of the decode workload for step ``step`` (position T0+step):
    q [B,H,D], q_I [B,H_I,D_I], w [B,H_I], and the new token's raw rows
    a, b, z [B,D], a_I, b_I, z_I [B,D_I], kv_raw [B,D].  Seeded by (seed, step)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed * 1000003 + step + 1)
    dt = _DT[cfg.dtype]
    B, H, D, HI, DI = cfg.B, cfg.H, cfg.D, cfg.HI, cfg.DI
    x = {}
    x["q"] = _draw(gen, (B, H, D), device, dt)
    x["q_I"] = _draw(gen, (B, HI, DI), device, dt)
    x["w"] = _draw(gen, (B, HI), device, torch.float32, kind="uniform")
    for name, dim in (("a", D), ("b", D), ("z", D), ("a_I", DI), ("b_I", DI), ("z_I", DI), ("kv_raw", D)):
        x[name] = _draw(gen, (B, dim), device, dt)
    return x
