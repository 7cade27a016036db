"""Layer drivers: one CSA or HCA prefill layer as a fixed sequence of C-ABI calls
on pre-allocated device buffers (every step of the path runs in the library's
kernels; this module only sequences the calls and owns the buffers).

CSA prefill (cf-1.com/news/5231315 §3.1, §3.3, §3.4):
    csa_compress(a, b, z)         -> kv_c  [B, S, D]
    csa_compress(a_I, b_I, z_I)   -> k_I   NVFP4 [B, S, D_I/2] + scales
    nvfp4_quantize(q_I)           -> q_I   NVFP4
    per chunk of query rows:
        indexer_score             -> score [B, Tc, S]
        topk_select               -> idx   [B, Tc, k]
        sparse_attn_fwd           -> out rows (window + sink fused)
HCA prefill (§3.2, §3.3):
    hca_compress(a, z)            -> kv_c  [B, S, D]
    hca_dense_attn_fwd            -> out
"""
from __future__ import annotations

import os

import torch

from . import ops

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def _no_timer(name):
    return _Null()


def _check_mode(check):
    return bool(int(os.environ.get("CSA_CHECK", "0"))) if check is None else bool(check)


def raise_on_status(status):
    """Raise if a check or a bounded wait recorded an error in ``status``."""
    v = int(status.item())
    if v != 0:
        status.zero_()
        raise ops.CsaError("device check", v & 0xFF)


class CsaPrefill:
    """Buffers + call sequence of one CSA prefill layer.  ``chunk`` bounds the
    query rows scored at once (the score buffer is [B, chunk, S])."""

    def __init__(self, cfg, device="cuda", chunk=None, gscale=1.0, fused=None, check=None):
        self.cfg = cfg
        c = cfg
        dt = _DT[c.dtype]
        self.sdt = torch.float32 if c.dtype == "f32" else torch.bfloat16
        self.chunk = min(c.T, chunk or c.T)
        self.g = gscale
        S = c.S
        # fused=True scores and selects in one kernel (indexer_topk: BF16 scores
        # whose rows fit on chip); by default the scores go through HBM
        # (indexer_score + topk_select), which is the faster of the two on the
        # 32K-token prefill shapes (0.59 ms against 0.62 ms on one B200)
        can_fuse = c.dtype == "bf16" and 0 < S <= ops.indexer_topk_max_entries(c.HI, c.DI)
        self.fused = bool(fused)
        if self.fused and not can_fuse:
            raise ValueError("indexer_topk does not support this layer shape")
        self.kv_c = torch.empty((c.B, S, c.D), dtype=dt, device=device)
        self.k_fp4 = torch.empty((c.B, S, c.DI // 2), dtype=torch.uint8, device=device)
        self.k_sf = torch.empty((c.B, S, c.DI // 16), dtype=torch.uint8, device=device)
        self.q_fp4 = torch.empty((c.B, c.T, c.HI, c.DI // 2), dtype=torch.uint8, device=device)
        self.q_sf = torch.empty((c.B, c.T, c.HI, c.DI // 16), dtype=torch.uint8, device=device)
        self.score = None if self.fused else torch.empty((c.B, self.chunk, S), dtype=self.sdt, device=device)
        self.idx = torch.empty((c.B, self.chunk, c.k), dtype=torch.int32, device=device)
        self.out = torch.empty((c.B, c.T, c.H, c.D), dtype=dt, device=device)
        self.lse = None
        self.q_pos0 = torch.zeros((c.B,), dtype=torch.int32, device=device)
        self.launches = 3 + (2 if self.fused else 3) * ((c.T + self.chunk - 1) // self.chunk)
        # check mode (argument, or CSA_CHECK=1 in the environment): every idx
        # chunk is bounds-checked before the attention gathers with it
        self.check = _check_mode(check)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device) if self.check else None
        self.launches += ((c.T + self.chunk - 1) // self.chunk) if self.check else 0

    def run(self, x, keep_idx=None, timer=None):
        """x: dict of device tensors (input generator order).  If ``keep_idx`` is a
        tensor [B, T, k] the selected indices of every chunk are copied into it.
        ``timer(name)`` may return a context manager wrapped around each call."""
        c = self.cfg
        t = timer or _no_timer
        with t("csa_compress"):
            ops.csa_compress(x["a"], x["b"], x["z"], c.m, out=self.kv_c)
        with t("csa_compress_indexer_keys"):
            ops.csa_compress(x["a_I"], x["b_I"], x["z_I"], c.m, out_fp4=self.k_fp4, out_sf=self.k_sf,
                             gscale=self.g, out_dtype=x["a_I"].dtype)
        with t("nvfp4_quantize"):
            ops.nvfp4_quantize(x["q_I"], self.q_fp4, self.q_sf, self.g)
        for r0 in range(0, c.T, self.chunk):
            tc = min(self.chunk, c.T - r0)
            ix = self.idx.view(-1)[: c.B * tc * c.k].view(c.B, tc, c.k)
            if self.fused:
                with t("indexer_topk"):
                    ops.indexer_topk(self.q_fp4, self.q_sf, self.k_fp4, self.k_sf, x["w"], self.q_pos0, ix, c.S,
                                     c.m, row0=r0, T_chunk=tc, q_gscale=self.g, k_gscale=self.g)
            else:
                sc = self.score.view(-1)[: c.B * tc * c.S].view(c.B, tc, c.S)
                with t("indexer_score"):
                    ops.indexer_score(self.q_fp4, self.q_sf, self.k_fp4, self.k_sf, x["w"], self.q_pos0, sc, c.S,
                                      c.m, row0=r0, T_chunk=tc, q_gscale=self.g, k_gscale=self.g)
                with t("topk_select"):
                    ops.topk_select(sc, ix, c.S, c.m, self.q_pos0, row0=r0)
            if self.check:
                ops.validate_indices(ix, c.S, c.m, self.q_pos0, self.status, row0=r0)
            with t("sparse_attn_fwd"):
                ops.sparse_attn_fwd(x["q"], self.kv_c, ix, x["kv_raw"], x["sink"], c.tau, c.W, self.q_pos0,
                                    self.out, self.lse, row0=r0, T_chunk=tc)
            if keep_idx is not None:
                keep_idx[:, r0:r0 + tc].copy_(ix)
        if self.check:
            raise_on_status(self.status)
        return self.out


class HcaPrefill:
    """Buffers + call sequence of one HCA prefill layer."""

    def __init__(self, cfg, device="cuda"):
        self.cfg = cfg
        c = cfg
        dt = _DT[c.dtype]
        self.kv_c = torch.empty((c.B, c.S, c.D), dtype=dt, device=device)
        self.out = torch.empty((c.B, c.T, c.H, c.D), dtype=dt, device=device)
        self.lse = None
        self.q_pos0 = torch.zeros((c.B,), dtype=torch.int32, device=device)
        self.launches = 2

    def run(self, x, timer=None):
        c = self.cfg
        t = timer or _no_timer
        with t("hca_compress"):
            ops.hca_compress(x["a"], x["z"], c.m, self.kv_c)
        with t("hca_dense_attn_fwd"):
            ops.hca_dense_attn_fwd(x["q"], self.kv_c, x["kv_raw"], x["sink"], c.tau, c.W, self.q_pos0, self.out,
                                   c.m, lse=self.lse)
        return self.out


_CARRY = ("a", "b", "z", "a_I", "b_I", "z_I")


class CsaDecode:
    """Buffers + call sequence of one CSA decode step: one new token for each of
    B sequences (cf-1.com/news/5231315 §3.1, §3.3; the cached state grows by one
    compressed entry every m tokens and the raw window is a W-slot ring).

    ``state`` is the synthetic cache at position T0 (``inputs.decode_state`` on
    the device): kv_c [B, cap, D], k_I_src [B, cap, D_I], ring [B, W, D] and the
    raw rows of the last complete block ``carry_*`` [B, m, dim].  The indexer keys
    of the cache are quantised to NVFP4 once here; per step:

        csa_ring_append x6            token p -> compressor carry slot p % 2m
        csa_compress (decode mode)    entry (p+1)/m - 1 when block completes -> kv_c
        csa_compress (decode, NVFP4)  the same entry's indexer key        -> k_I
        csa_ring_append               token p's raw KV -> ring slot p % W
        nvfp4_quantize                q_I
          (these five lines are one csa_decode_update launch for bf16 caches)
        indexer_score                 score [B, 1, cap] (visible prefix only)
        topk_select                   idx [B, 1, k] (multi-CTA rows, workspace)
        sparse_attn_fwd               out [B, 1, H, D] (window + sink fused)
        csa_pos_advance               p += 1 on the device

    Every launch reads the position from device memory, so the step can be
    captured once in a CUDA graph (``capture``) and replayed.
    """

    def __init__(self, cfg, state, T0, device="cuda", gscale=1.0, with_lse=False, fused_update=None, check=None):
        self.cfg = c = cfg
        dt = _DT[c.dtype]
        self.dt = dt
        self.g = gscale
        self.T0 = T0
        self.kv_c = state["kv_c"]
        B, cap, D = self.kv_c.shape
        self.cap = cap
        if "k_fp4" in state:
            # keys already quantised (a cache restored from a prefill)
            self.k_fp4, self.k_sf = state["k_fp4"], state["k_sf"]
        else:
            self.k_fp4 = torch.empty((B, cap, c.DI // 2), dtype=torch.uint8, device=device)
            self.k_sf = torch.empty((B, cap, c.DI // 16), dtype=torch.uint8, device=device)
            ops.nvfp4_quantize(state["k_I_src"], self.k_fp4, self.k_sf, gscale)
        self.ring = state["ring"]
        self.carry = {}
        slot0 = ((T0 // c.m - 1) % 2) * c.m      # the last complete block's slots
        for n in _CARRY:
            if "carry_ring_" + n in state:
                # a full 2m-slot carry ring (token j at slot j % 2m)
                self.carry[n] = state["carry_ring_" + n]
                continue
            src = state["carry_" + n]
            buf = torch.zeros((B, 2 * c.m, src.shape[-1]), dtype=dt, device=device)
            buf[:, slot0:slot0 + c.m] = src
            self.carry[n] = buf
        self.pos = torch.full((B,), T0, dtype=torch.int32, device=device)
        self.q_fp4 = torch.empty((B, 1, c.HI, c.DI // 2), dtype=torch.uint8, device=device)
        self.q_sf = torch.empty((B, 1, c.HI, c.DI // 16), dtype=torch.uint8, device=device)
        sdt = torch.float32 if c.dtype == "f32" else torch.bfloat16
        # row stride padded to 8 elements so every score row is 16-byte aligned
        self.score = torch.empty((B, 1, (cap + 7) // 8 * 8), dtype=sdt, device=device)
        self.idx = torch.empty((B, 1, c.k), dtype=torch.int32, device=device)
        self.out = torch.empty((B, 1, c.H, D), dtype=dt, device=device)
        self.lse = torch.empty((B, 1, c.H), dtype=torch.float32, device=device) if with_lse else None
        nws = ops.topk_workspace_size(B, 1, cap, c.k)
        self.ws = torch.empty((max(1, nws // 4),), dtype=torch.int32, device=device) if nws else None
        self.sink = state.get("sink")
        # the cache update of a step (7 appends, 2 compressions, the q_I
        # quantisation) in one launch where the shapes allow (bf16)
        can_fuse = c.dtype == "bf16" and c.D % 16 == 0 and c.DI % 16 == 0 and c.DI <= 256
        self.fused_update = can_fuse if fused_update is None else bool(fused_update)
        # multi-CTA top-k: workspace memset + three kernels
        self.launches = (1 if self.fused_update else 6 + 2 + 1 + 1) + 1 + (4 if nws else 1) + 1 + 1
        # check mode: idx is bounds-checked on the device every step; the
        # caller reads the verdict with raise_on_status(self.status)
        self.check = _check_mode(check)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device) if self.check else None
        self.launches += 1 if self.check else 0
        self.graph = None
        self.x = None

    def step(self, x, timer=None):
        """x: per-step device inputs (``inputs.decode_step_inputs`` layout, plus
        ``sink`` [H] if the state has none).  Returns out [B, 1, H, D]."""
        c = self.cfg
        t = timer or _no_timer
        if self.fused_update:
            with t("csa_decode_update"):
                ops.csa_decode_update(x, self.carry, self.ring, self.kv_c, self.k_fp4, self.k_sf, self.q_fp4,
                                      self.q_sf, self.pos, c.m, self.g)
        else:
            for n in _CARRY:
                with t("csa_ring_append"):
                    ops.csa_ring_append(x[n], self.carry[n], self.pos)
            with t("csa_compress"):
                ops.csa_compress(self.carry["a"], self.carry["b"], self.carry["z"], c.m, out=self.kv_c,
                                 ring_pos=self.pos, out_bstride=self.cap)
            with t("csa_compress_indexer_keys"):
                ops.csa_compress(self.carry["a_I"], self.carry["b_I"], self.carry["z_I"], c.m,
                                 out_fp4=self.k_fp4, out_sf=self.k_sf, gscale=self.g, ring_pos=self.pos,
                                 out_bstride=self.cap, out_dtype=self.dt)
            with t("csa_ring_append"):
                ops.csa_ring_append(x["kv_raw"], self.ring, self.pos)
            with t("nvfp4_quantize"):
                ops.nvfp4_quantize(x["q_I"], self.q_fp4, self.q_sf, self.g)
        with t("indexer_score"):
            ops.indexer_score(self.q_fp4, self.q_sf, self.k_fp4, self.k_sf, x["w"].view(-1, 1, c.HI), self.pos,
                              self.score, self.cap, c.m, q_gscale=self.g, k_gscale=self.g)
        with t("topk_select"):
            ops.topk_select(self.score, self.idx, self.cap, c.m, self.pos, workspace=self.ws)
        if self.check:
            ops.validate_indices(self.idx, self.cap, c.m, self.pos, self.status)
        sink = x["sink"] if "sink" in x else self.sink
        with t("sparse_attn_fwd"):
            ops.sparse_attn_fwd(x["q"].view(-1, 1, c.H, x["q"].shape[-1]), self.kv_c, self.idx, self.ring, sink,
                                c.tau, c.W, self.pos, self.out, self.lse, raw_cap=c.W)
        with t("csa_pos_advance"):
            ops.csa_pos_advance(self.pos, 1)
        return self.out

    def capture(self, x):
        """Record one step on static input buffers ``x`` into a CUDA graph; the
        caller refills ``x`` in place and calls ``replay``.  Run ``step`` once
        before capturing (first-call set-up such as kernel attributes must not
        happen inside the capture), and note that capture itself does not
        advance the position."""
        self.x = x
        p0 = self.pos.clone()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.step(x)
        torch.cuda.current_stream().wait_stream(s)
        self.pos.copy_(p0)
        self.graph = g
        return g

    def replay(self):
        self.graph.replay()
        return self.out


class PrefixCheckpoints:
    """Periodic snapshots of a CSA layer's decode-time state, taken from the
    inputs of a prefill (cf-1.com/news/5231315 §4.4: the sliding-window cache
    is checkpointed every 1024 tokens, so a request that shares a prefix
    restores that state instead of recomputing it).

    Snapshot c covers the tokens up to p_c = every * (c + 1) - 1 and holds the
    raw window ring [B, n, W, D] and, for each compressor stream, the carry
    ring [B, n, 2m, dim] (the last complete block and the block in progress),
    in the decode layout (token j at slot j % cap).  The compressed entries and
    NVFP4 keys of the prefix are not copied: once emitted they are final, so
    the prefill's own buffers serve every snapshot (entries s < (p_c + 1) / m).
    One ``csa_state_gather`` launch per tensor builds all snapshots."""

    def __init__(self, cfg, x, every=1024, device="cuda"):
        c = cfg
        self.cfg, self.every = cfg, every
        n = c.T // every
        self.positions = [every * (i + 1) - 1 for i in range(n)]
        self.pos = torch.tensor([self.positions] * c.B, dtype=torch.int32, device=device)
        dt = x["kv_raw"].dtype
        self.ring = torch.empty((c.B, n, c.W, c.D), dtype=dt, device=device)
        ops.csa_state_gather(x["kv_raw"], self.pos, self.ring, m=0, nrows=c.W)
        self.carry = {}
        for name in _CARRY:
            src = x[name]
            buf = torch.empty((c.B, n, 2 * c.m, src.shape[-1]), dtype=dt, device=device)
            ops.csa_state_gather(src, self.pos, buf, m=c.m)
            self.carry[name] = buf
        self.launches = 1 + len(_CARRY)

    def restore(self, dcfg, i, kv_c, k_fp4, k_sf, extra_entries, device="cuda", with_lse=False):
        """A CsaDecode positioned after snapshot i (next token p_i + 1), with a
        cache of the prefix's entries plus room for ``extra_entries`` more."""
        p = self.positions[i]
        n_ent = (p + 1) // dcfg.m
        B = kv_c.shape[0]
        cap = n_ent + extra_entries
        st = {"kv_c": torch.zeros((B, cap, kv_c.shape[-1]), dtype=kv_c.dtype, device=device),
              "k_fp4": torch.zeros((B, cap, k_fp4.shape[-1]), dtype=torch.uint8, device=device),
              "k_sf": torch.zeros((B, cap, k_sf.shape[-1]), dtype=torch.uint8, device=device),
              "ring": self.ring[:, i].contiguous()}
        st["kv_c"][:, :n_ent] = kv_c[:, :n_ent]
        st["k_fp4"][:, :n_ent] = k_fp4[:, :n_ent]
        st["k_sf"][:, :n_ent] = k_sf[:, :n_ent]
        for name in _CARRY:
            st["carry_ring_" + name] = self.carry[name][:, i].contiguous()
        return CsaDecode(dcfg, st, p + 1, device=device, with_lse=with_lse)


class Stack:
    """An interleaved prefill stack: the layers of ``cfgs`` (e.g. HCA, HCA, CSA,
    CSA, as in the [attention.hca] interleave_pattern of yfxerp.com/news/211352
    §3) run one after another, each on its own inputs; the layers do not feed
    each other (no projections or residual path are part of this layer)."""

    def __init__(self, cfgs, device="cuda", chunk=16384):
        self.layers = []
        for c in cfgs:
            self.layers.append(CsaPrefill(c, device=device, chunk=chunk) if c.kind == "csa"
                               else HcaPrefill(c, device=device))
        self.launches = sum(lay.launches for lay in self.layers)

    def run(self, xs, timer=None):
        """xs: one input dict per layer.  Returns the layers' outputs."""
        return [lay.run(x, timer=timer) for lay, x in zip(self.layers, xs)]
