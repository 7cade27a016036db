"""Prefill of one sequence split over ranks (one process per GPU).

The query rows of a CSA prefill layer are cut into contiguous shards whose
sizes are multiples of the compression ratio m, so every compressed block lies
in one shard.  Rank r, owning tokens [start_r, end_r):

  1. compresses its own blocks.  The first entry of a shard mixes the last
     block of the left neighbour (the overlap of cf-1.com/news/5231315 §3.1),
     so the m raw rows of that block come over as a halo, and the compressor
     runs with first_has_pred = 1;
  2. all-gathers the compressed entries and their NVFP4 indexer keys: a query
     at position p sees every completed block before it, wherever it was
     compressed (one collective per layer, a few MB);
  3. quantises its own q_I, scores its rows against all entries, selects the
     top-k and attends.  The raw window of its first W - 1 rows reaches into
     the left neighbour's tokens, which come over as a second halo; the window
     rows are laid out as a ring (token j at slot j % raw_cap) so the attention
     kernel reads them by absolute position.

Every step of the layer runs in the library's kernels (``ops``); this module
only plans the shards, moves the halos and the entries between ranks
(torch.distributed), and assembles the ring.
"""
from __future__ import annotations

import torch

from . import ops

_STREAMS = ("a", "b", "z", "a_I", "b_I", "z_I")


class ShardPlan:
    """Token ranges of ``world`` shards of a T-token sequence: blocks of m
    tokens are split as evenly as possible (earlier ranks take the extra
    blocks); the trailing partial block, which emits no entry, goes to the
    last rank."""

    def __init__(self, T: int, m: int, W: int, world: int):
        self.T, self.m, self.W, self.world = T, m, W, world
        blocks = T // m
        base, extra = divmod(blocks, world)
        self.start, self.end = [], []
        s = 0
        for r in range(world):
            n = (base + (1 if r < extra else 0)) * m
            self.start.append(s)
            s += n
            self.end.append(s)
        self.end[-1] = T

    def rows(self, r):
        return self.start[r], self.end[r]

    def entries(self, r):
        """Compressed entries rank r emits: blocks [start/m, end/m)."""
        return self.start[r] // self.m, self.end[r] // self.m

    def raw_halo(self, r):
        """Raw tokens before the shard that its rows' windows reach."""
        s = self.start[r]
        return max(0, s - (self.W - 1)), s


# ----------------------------------------------------------------- exchange
def left_halo(t_local, n, group=None):
    """Every rank sends the last ``n`` rows (dim 1) of its shard to the next
    rank; returns the rows received from the previous rank (rank 0: zero rows).
    Implemented as one all-gather of the n-row tails."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    tail = t_local[:, t_local.shape[1] - n:].contiguous()
    parts = [torch.empty_like(tail) for _ in range(world)]
    dist.all_gather(parts, tail, group=group)
    if rank == 0:
        return tail[:, :0]
    return parts[rank - 1]


def gather_entries(e_local, counts, group=None):
    """All-gather of per-rank entry blocks of sizes ``counts`` along dim 1
    (padded to the largest count for the collective), concatenated in rank
    order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n_max = max(counts)
    pad = torch.zeros((e_local.shape[0], n_max) + tuple(e_local.shape[2:]), dtype=e_local.dtype,
                      device=e_local.device)
    pad[:, :e_local.shape[1]] = e_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :c] for p, c in zip(parts, counts)], dim=1)


# ------------------------------------------------------------- shard layer
class CsaPrefillShard:
    """One rank's part of a CSA prefill layer (see the module docstring).
    ``x`` holds the rank's rows [start, end) of every input stream (plus the
    sink); halos are passed in by the caller, who moves them between ranks."""

    def __init__(self, cfg, plan: ShardPlan, rank: int, device="cuda", gscale=1.0):
        self.cfg, self.plan, self.rank, self.g = cfg, plan, rank, gscale
        self.start, self.end = plan.rows(rank)
        self.device = device
        self.q_pos0 = torch.full((cfg.B,), self.start, dtype=torch.int32, device=device)

    def compress(self, x, pred):
        """Entries of the rank's own blocks.  ``pred``: the m raw rows of the
        left neighbour's last block for each compressor stream (rank 0: empty).
        Returns kv_c [B, n, D], k_fp4 [B, n, D_I/2], k_sf [B, n, D_I/16]."""
        c = self.cfg
        e0, e1 = self.plan.entries(self.rank)
        n = e1 - e0
        fhp = 1 if self.rank > 0 else 0
        src = {s: (torch.cat([pred[s], x[s]], dim=1) if fhp else x[s]).contiguous() for s in _STREAMS}
        kv = torch.empty((c.B, n, c.D), dtype=x["a"].dtype, device=self.device)
        k4 = torch.empty((c.B, n, c.DI // 2), dtype=torch.uint8, device=self.device)
        ksf = torch.empty((c.B, n, c.DI // 16), dtype=torch.uint8, device=self.device)
        if n > 0:
            ops.csa_compress(src["a"], src["b"], src["z"], c.m, out=kv, first_has_pred=fhp)
            ops.csa_compress(src["a_I"], src["b_I"], src["z_I"], c.m, out_fp4=k4, out_sf=ksf, gscale=self.g,
                             first_has_pred=fhp, out_dtype=x["a_I"].dtype)
        return kv, k4, ksf

    def attend(self, x, raw_halo, kv_c, k_fp4, k_sf):
        """Score, select and attend for the rank's rows against all entries
        (kv_c, k_fp4, k_sf [B, S, .] in entry order).  ``raw_halo``: kv_raw rows
        [max(0, start - W + 1), start) from the left neighbour.  Returns
        out [B, end - start, H, D]."""
        c = self.cfg
        Tl = self.end - self.start
        S = kv_c.shape[1]
        q_fp4 = torch.empty((c.B, Tl, c.HI, c.DI // 2), dtype=torch.uint8, device=self.device)
        q_sf = torch.empty((c.B, Tl, c.HI, c.DI // 16), dtype=torch.uint8, device=self.device)
        ops.nvfp4_quantize(x["q_I"], q_fp4, q_sf, self.g)
        sdt = torch.float32 if c.dtype == "f32" else torch.bfloat16
        score = torch.empty((c.B, Tl, max(S, 1)), dtype=sdt, device=self.device)
        idx = torch.empty((c.B, Tl, c.k), dtype=torch.int32, device=self.device)
        if S > 0:
            ops.indexer_score(q_fp4, q_sf, k_fp4, k_sf, x["w"], self.q_pos0, score, S, c.m, q_gscale=self.g,
                              k_gscale=self.g)
        ops.topk_select(score, idx, S, c.m, self.q_pos0)
        ring = window_ring(raw_halo, x["kv_raw"], self.start, c.W)
        raw_cap = ring.shape[1]
        out = torch.empty((c.B, Tl, c.H, c.D), dtype=x["q"].dtype, device=self.device)
        ops.sparse_attn_fwd(x["q"], kv_c if S > 0 else torch.zeros((c.B, 1, c.D), dtype=x["q"].dtype,
                                                                       device=self.device),
                            idx, ring, x["sink"], c.tau, c.W, self.q_pos0, out, raw_cap=raw_cap)
        return out


def window_ring(raw_halo, kv_raw_local, start, W):
    """The raw rows a shard's windows read, as a ring: token j at slot
    j % raw_cap for j in [start - halo, end), raw_cap = max(W, rows) so no two
    tokens collide and the attention's ring indexing finds every window row."""
    lo = start - raw_halo.shape[1]
    seq = torch.cat([raw_halo, kv_raw_local], dim=1)
    if seq.shape[1] < W:
        pad = torch.zeros((seq.shape[0], W - seq.shape[1]) + tuple(seq.shape[2:]), dtype=seq.dtype,
                          device=seq.device)
        seq = torch.cat([seq, pad], dim=1)
    return torch.roll(seq, shifts=lo % seq.shape[1], dims=1).contiguous()


def shard_inputs(x, plan: ShardPlan, r: int):
    """Rank r's rows of a full input dict, and its halos (for tests and for a
    driver that holds the whole sequence)."""
    s, e = plan.rows(r)
    xl = {k: (v if k == "sink" else v[:, s:e].contiguous()) for k, v in x.items()}
    m = plan.m
    pred = {n: x[n][:, max(0, s - m):s].contiguous() for n in _STREAMS}
    h0, h1 = plan.raw_halo(r)
    raw_halo = x["kv_raw"][:, h0:h1].contiguous()
    return xl, pred, raw_halo


def run_rank(cfg, x_local, plan: ShardPlan, rank: int, group=None, device="cuda"):
    """One rank's whole prefill layer under torch.distributed: both halos and
    the entry all-gather over ``group``, the kernels on this rank's GPU.
    ``x_local``: this rank's rows of every stream (and the sink).  Returns
    out [B, end - start, H, D] for the rank's rows."""
    lay = CsaPrefillShard(cfg, plan, rank, device=device)
    pred = {n: left_halo(x_local[n], cfg.m, group) for n in _STREAMS}
    raw_halo = left_halo(x_local["kv_raw"], cfg.W - 1, group)
    h0, h1 = plan.raw_halo(rank)
    raw_halo = raw_halo[:, raw_halo.shape[1] - (h1 - h0):]
    kv, k4, ksf = lay.compress(x_local, pred)
    counts = [plan.entries(r)[1] - plan.entries(r)[0] for r in range(plan.world)]
    kv_c = gather_entries(kv, counts, group)
    k_fp4 = gather_entries(k4, counts, group)
    k_sf = gather_entries(ksf, counts, group)
    return lay.attend(x_local, raw_halo, kv_c, k_fp4, k_sf)
