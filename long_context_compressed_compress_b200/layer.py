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


class CsaPrefill:
    """Buffers + call sequence of one CSA prefill layer.  ``chunk`` bounds the
    query rows scored at once (the score buffer is [B, chunk, S])."""

    def __init__(self, cfg, device="cuda", chunk=None, gscale=1.0):
        self.cfg = cfg
        c = cfg
        dt = _DT[c.dtype]
        self.sdt = torch.float32 if c.dtype == "f32" else torch.bfloat16
        self.chunk = min(c.T, chunk or c.T)
        self.g = gscale
        S = c.S
        self.kv_c = torch.empty((c.B, S, c.D), dtype=dt, device=device)
        self.k_fp4 = torch.empty((c.B, S, c.DI // 2), dtype=torch.uint8, device=device)
        self.k_sf = torch.empty((c.B, S, c.DI // 16), dtype=torch.uint8, device=device)
        self.q_fp4 = torch.empty((c.B, c.T, c.HI, c.DI // 2), dtype=torch.uint8, device=device)
        self.q_sf = torch.empty((c.B, c.T, c.HI, c.DI // 16), dtype=torch.uint8, device=device)
        self.score = torch.empty((c.B, self.chunk, S), dtype=self.sdt, device=device)
        self.idx = torch.empty((c.B, self.chunk, c.k), dtype=torch.int32, device=device)
        self.out = torch.empty((c.B, c.T, c.H, c.D), dtype=dt, device=device)
        self.lse = None
        self.q_pos0 = torch.zeros((c.B,), dtype=torch.int32, device=device)
        self.launches = 3 + 3 * ((c.T + self.chunk - 1) // self.chunk)

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
            sc = self.score.view(-1)[: c.B * tc * c.S].view(c.B, tc, c.S)
            ix = self.idx.view(-1)[: c.B * tc * c.k].view(c.B, tc, c.k)
            with t("indexer_score"):
                ops.indexer_score(self.q_fp4, self.q_sf, self.k_fp4, self.k_sf, x["w"], self.q_pos0, sc, c.S, c.m,
                                  row0=r0, T_chunk=tc, q_gscale=self.g, k_gscale=self.g)
            with t("topk_select"):
                ops.topk_select(sc, ix, c.S, c.m, self.q_pos0, row0=r0)
            with t("sparse_attn_fwd"):
                ops.sparse_attn_fwd(x["q"], self.kv_c, ix, x["kv_raw"], x["sink"], c.tau, c.W, self.q_pos0,
                                    self.out, self.lse, row0=r0, T_chunk=tc)
            if keep_idx is not None:
                keep_idx[:, r0:r0 + tc].copy_(ix)
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
