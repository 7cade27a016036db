"""Plain CPU oracle of the CSA / HCA compressed long-context attention layer.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct statement
of what the GPU library computes.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it; the product path never does, and it shares no code with the CUDA kernels.

Arithmetic is float64 throughout (numpy), with exactly one rounding to the
storage type at each storage point (compressed entries, scores, outputs), except
the NVFP4 quantiser, whose scale and quotient steps are defined in fp32.

Sources (web pages describing the DeepSeek-V4 attention design):
  [cf-1]   cf-1.com/news/5231315 "企业官网建设流程全解析" (page title as served), a
           DeepSeek-V4 write-up: §3.1 "CSA 的工作方式", §3.2 "HCA 的工作方式",
           §3.3 "层间排布与滑窗补充", §3.4 "两个降开销的设计",
           §4.3 "确定性 Kernel", §4.4 "FP4 QAT 与 KV Cache 层级".
  [yfxerp] yfxerp.com/news/211352 "DeepSeek-V4 原理拆解：百万上下文之外，
           CSA/HCA/mHC/MegaMoE 强在哪", §1 and the §3 "config.toml" skeleton
           ([attention.csa] / [attention.hca] blocks).
  [csdn-b] devpress.csdn.net/awstech/6a4623aa…, §2.2 "注意力机制的颠覆".

Where those pages leave a formula open, the oracle takes these readings
(each one is listed with its justification in the design notes):
  * CSA gate: per channel, one softmax over the 2m gate logits z of the current
    block and its predecessor; the current block mixes stream ``a``, the
    predecessor block mixes stream ``b`` ("two independent KV sequences ...
    softmax-normalised gate weights ... adjacent blocks share indices", [cf-1] §3.1).
    Entry 0 has no predecessor: its softmax runs over the m current logits only.
  * HCA gate: per channel, a softmax over the block's m logits mixing ``a``
    ([cf-1] §3.2, 128 tokens per entry, no overlap).
  * A trailing partial block emits no entry; entry s is visible to the query at
    absolute position p iff m*(s+1) - 1 <= p (only completed blocks).
  * Indexer: score[t,s] = sum_h w[t,h] * ReLU(qhat[t,h,:] . khat[s,:]) with
    qhat, khat the NVFP4-dequantised values ([cf-1] §3.4 FP4 QK).
  * Top-k: the k largest visible scores, ties to the smaller index, emitted in
    ascending index order, padded with -1.
  * Attention: MQA, one shared KV head, key = value = the entry (or raw token)
    vector; the sliding window holds raw tokens j with p-W < j <= p, j >= 0
    ([cf-1] §3.3, W = 128); the sink logit sigma_h adds exp(sigma_h) to the
    softmax denominator only ([cf-1] §3.3: a learnable term added to the denominator).
    lse is the log-sum-exp of the logits without the sink.
"""
from __future__ import annotations

import numpy as np

from . import formats

__all__ = [
    "csa_compress", "hca_compress", "nvfp4_quantize", "visible_entries",
    "indexer_score", "round_scores", "topk_select", "attend_rows",
    "sparse_attn", "dense_attn", "swa_sink_merge", "round_out",
    "csa_layer", "hca_layer", "csa_decode_step", "grouped_out_proj",
]


def _f64(x):
    """Host tensor/array -> float64 numpy array (exact for fp32 / bf16 inputs)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# (1) compressors
# ---------------------------------------------------------------------------

def csa_compress(a, b, z, m: int = 4, first_has_pred: bool = False):
    """Overlapping gated m:1 compression ([cf-1] §3.1; [yfxerp] §1: the KV of every
    4 adjacent tokens becomes one entry; kv_compress_ratio 4 in the [attention.csa] block).

    a, b, z: [..., T, D].  Returns e: [..., S, D] float64 (unrounded), where
    S = T // m, or T // m - 1 when ``first_has_pred`` (then rows [0, m) are only
    the predecessor block of the first emitted entry: the decode-time window).

    For entry i with current block C = rows [m*i, m*i+m) and predecessor
    P = rows [m*(i-1), m*i):
        alpha = softmax over the 2m values {z[t,c] : t in P u C}  (per channel c)
        e[i,c] = sum_{t in C} alpha_t a[t,c] + sum_{t in P} alpha_t b[t,c]
    Entry 0 without a predecessor: softmax over its m current logits only.
    """
    a, b, z = _f64(a), _f64(b), _f64(z)
    T, D = a.shape[-2], a.shape[-1]
    nblk = T // m
    lead = a.shape[:-2]
    ab = a[..., : nblk * m, :].reshape(*lead, nblk, m, D)
    bb = b[..., : nblk * m, :].reshape(*lead, nblk, m, D)
    zb = z[..., : nblk * m, :].reshape(*lead, nblk, m, D)
    out = []
    start = 1 if first_has_pred else 0
    for i in range(start, nblk):
        if i == 0:
            logits = zb[..., 0, :, :]                     # [..., m, D]
            vals = ab[..., 0, :, :]
        else:
            logits = np.concatenate([zb[..., i - 1, :, :], zb[..., i, :, :]], axis=-2)
            vals = np.concatenate([bb[..., i - 1, :, :], ab[..., i, :, :]], axis=-2)
        mx = logits.max(axis=-2, keepdims=True)
        wts = np.exp(logits - mx)
        wts = wts / wts.sum(axis=-2, keepdims=True)
        out.append((wts * vals).sum(axis=-2))
    if not out:
        return np.zeros((*lead, 0, D))
    return np.stack(out, axis=-2)


def hca_compress(a, z, m: int = 128):
    """Non-overlapping gated m:1 pooling ([cf-1] §3.2: one entry per 128 tokens;
    compress_ratio 128 in the [attention.hca] block of [yfxerp] §3).

    e[i,c] = sum_{t in block i} softmax_{t in block i}(z[t,c]) * a[t,c]
    """
    a, z = _f64(a), _f64(z)
    T, D = a.shape[-2], a.shape[-1]
    S = T // m
    lead = a.shape[:-2]
    ab = a[..., : S * m, :].reshape(*lead, S, m, D)
    zb = z[..., : S * m, :].reshape(*lead, S, m, D)
    mx = zb.max(axis=-2, keepdims=True)
    wts = np.exp(zb - mx)
    wts = wts / wts.sum(axis=-2, keepdims=True)
    return (wts * ab).sum(axis=-2)


# ---------------------------------------------------------------------------
# (2) NVFP4 quantisation of the indexer QK path
# ---------------------------------------------------------------------------

def nvfp4_quantize(x, g: float = 1.0):
    """NVFP4 block quantisation along the last dim, blocks of 16 ([cf-1] §3.4: the
    indexer's QK runs in FP4; §4.4 FP4 QK path; 16-element blocks with E4M3 scales).

    For block j with amax_j = max |x| (x taken as fp32):
        s_j  = E4M3_rne_sat( fp32( amax_j / fp32(6*g) ) )
        q    = E2M1_rne_sat( fp32( x / fp32(s_j * g) ) )      (q = +0 when s_j = 0)
        xhat = q * s_j * g
    All divisions and products here are single fp32 operations (IEEE RNE).

    Returns dict with float64 ``xhat``, E2M1 ``codes`` (one nibble per element),
    ``packed`` bytes (element 2i in the low nibble, 2i+1 in the high nibble) and
    E4M3 ``sf`` bytes, one per block.
    """
    x32 = np.asarray(_f64(x), dtype=np.float64).astype(np.float32)
    *lead, D = x32.shape
    if D % 16:
        raise ValueError("NVFP4 needs the last dim to be a multiple of 16")
    xb = x32.reshape(*lead, D // 16, 16)
    g32 = np.float32(g)
    amax = np.abs(xb).max(axis=-1)                                # fp32, exact
    s = formats.e4m3((amax / (np.float32(6.0) * g32)).astype(np.float64))
    denom = (s.astype(np.float32) * g32)[..., None]               # fp32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        quot = (xb / denom).astype(np.float64)                    # fp32 quotient
    q = np.where((s > 0)[..., None], formats.e2m1(quot), 0.0)
    xhat = q * s[..., None] * np.float64(g32)
    codes = formats.e2m1_code(q).reshape(*lead, D)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return {
        "xhat": xhat.reshape(*lead, D),
        "codes": codes,
        "packed": packed,
        "sf": formats.e4m3_code(s),
        "scale": s,
    }


# ---------------------------------------------------------------------------
# (3) lightning-indexer score and top-k
# ---------------------------------------------------------------------------

def visible_entries(p, m: int):
    """Number of compressed entries visible at absolute position p: entry s is
    visible iff m*(s+1) - 1 <= p, i.e. s < (p + 1) // m (completed blocks only)."""
    return (np.asarray(p, dtype=np.int64) + 1) // m


def indexer_score(qhat, khat, w, positions, m: int):
    """score[b,t,s] = sum_h w[b,t,h] * max(0, sum_c qhat[b,t,h,c] * khat[b,s,c])
    for visible s, NaN elsewhere ([cf-1] §3.1 lightning indexer, §3.4).

    qhat [B,T,H,Dc], khat [B,S,Dc], w [B,T,H], positions [B,T] (absolute p).
    Exact float64 values; see ``round_scores`` for the stored dtype.
    """
    qhat, khat, w = _f64(qhat), _f64(khat), _f64(w)
    dots = np.einsum("bthc,bsc->bths", qhat, khat)
    score = np.einsum("bth,bths->bts", w, np.maximum(dots, 0.0))
    S = khat.shape[1]
    vis = visible_entries(positions, m)                            # [B,T]
    mask = np.arange(S)[None, None, :] < vis[..., None]
    return np.where(mask, score, np.nan)


def round_scores(score, dtype: str):
    """Round exact scores once to the stored type: 'f32' or 'bf16' (RNE); the
    index scores are stored in BF16 ([cf-1] §4.4: the score is narrowed from FP32 to BF16)."""
    return formats.bf16(score) if dtype == "bf16" else formats.f32(score)


def topk_select(score, positions, m: int, k: int):
    """Per row, the k largest visible scores; ties go to the smaller entry index;
    indices are emitted ascending and padded with -1.  If fewer than k entries are
    visible, all of them are returned ([cf-1] §3.1: each query picks its top-k
    compressed entries; top_k_blocks in the [attention.csa] block of [yfxerp] §3).

    score [B,T,S] (values as stored, compared exactly; +0 and -0 are equal).
    Returns int32 [B,T,k].
    """
    score = np.asarray(score, dtype=np.float64)
    B, T, S = score.shape
    vis = visible_entries(positions, m)
    idx = np.full((B, T, k), -1, dtype=np.int32)
    for bi in range(B):
        for t in range(T):
            n = int(min(vis[bi, t], S))
            if n <= 0:
                continue
            row = score[bi, t, :n] + 0.0                 # -0 -> +0
            if n <= k:
                chosen = np.arange(n)
            else:
                # primary key: score descending; secondary: index ascending
                order = np.lexsort((np.arange(n), -row))
                chosen = np.sort(order[:k])
            idx[bi, t, : len(chosen)] = chosen
    return idx


# ---------------------------------------------------------------------------
# (4) attention with sliding window and sink
# ---------------------------------------------------------------------------

def attend_rows(qrow, keys, sink, tau: float):
    """Softmax attention of all heads of one query token over a key set.

    qrow [H,D], keys [J,D] (key = value, MQA), sink [H] (-inf for none).
        l_j = tau * <q_h, key_j>,  M = max(sigma_h, max_j l_j)
        out_h = sum_j e^{l_j - M} key_j / (e^{sigma_h - M} + sum_j e^{l_j - M})
        lse_h = log sum_j e^{l_j}           (sink excluded)
    An empty key set gives out = 0 and lse = -inf.
    """
    H = qrow.shape[0]
    sink = np.broadcast_to(np.asarray(sink, dtype=np.float64), (H,))
    if keys.shape[0] == 0:
        return np.zeros_like(qrow), np.full(H, -np.inf)
    logits = tau * (qrow @ keys.T)                                   # [H,J]
    lmax = logits.max(axis=1)
    M = np.maximum(sink, lmax)
    p = np.exp(logits - M[:, None])
    denom = np.exp(sink - M) + p.sum(axis=1)
    out = (p @ keys) / denom[:, None]
    lse = lmax + np.log(np.exp(logits - lmax[:, None]).sum(axis=1))
    return out, lse


def _window_rows(kv_raw_b, raw_cap: int, p: int, W: int):
    """Raw tokens j with p - W < j <= p, j >= 0, read from slot j % raw_cap."""
    lo = max(0, p - W + 1)
    js = np.arange(lo, p + 1)
    return kv_raw_b[js % raw_cap]


def sparse_attn(q, kv_c, idx, kv_raw, raw_cap, sink, tau, W, positions, rows=None):
    """CSA attention: each query attends to its selected entries (idx != -1) plus
    the raw-token window, with the sink ([cf-1] §3.1 and §3.3).

    q [B,T,H,D], kv_c [B,S,D], idx [B,T,k], kv_raw [B,raw_cap,D], sink [H] or None,
    positions [B,T].  ``rows`` optionally restricts the evaluation to a list of
    (b, t) pairs (returned in that order).  Returns float64 out, lse.
    """
    kv_c, kv_raw = _f64(kv_c), _f64(kv_raw)     # q is converted row by row
    if not isinstance(idx, dict):               # a dict maps (b, t) -> that row's idx
        idx = np.asarray(idx)
    H = q.shape[2]
    snk = np.full(H, -np.inf) if sink is None else _f64(sink)
    pos = np.asarray(positions)
    pairs = rows if rows is not None else [(b, t) for b in range(q.shape[0]) for t in range(q.shape[1])]
    outs, lses = [], []
    for (b, t) in pairs:
        ir = np.asarray(idx[(b, t)])
        sel = ir[ir >= 0]
        keys = kv_c[b, sel]
        if W > 0:
            keys = np.concatenate([keys, _window_rows(kv_raw[b], raw_cap, int(pos[b, t]), W)], axis=0)
        o, l = attend_rows(_f64(q[b, t]), keys, snk, tau)
        outs.append(o)
        lses.append(l)
    return _reshape_rows(outs, lses, q, rows)


def dense_attn(q, kv_c, kv_raw, raw_cap, sink, tau, W, positions, m, rows=None):
    """HCA attention: each query attends to every visible compressed entry
    ([cf-1] §3.2: no sparse selection, dense attention) plus the raw window and sink."""
    kv_c, kv_raw = _f64(kv_c), _f64(kv_raw)     # q is converted row by row
    H = q.shape[2]
    snk = np.full(H, -np.inf) if sink is None else _f64(sink)
    pos = np.asarray(positions)
    pairs = rows if rows is not None else [(b, t) for b in range(q.shape[0]) for t in range(q.shape[1])]
    outs, lses = [], []
    for (b, t) in pairs:
        p = int(pos[b, t])
        n = int(min(visible_entries(p, m), kv_c.shape[1]))
        keys = kv_c[b, :n]
        if W > 0:
            keys = np.concatenate([keys, _window_rows(kv_raw[b], raw_cap, p, W)], axis=0)
        o, l = attend_rows(_f64(q[b, t]), keys, snk, tau)
        outs.append(o)
        lses.append(l)
    return _reshape_rows(outs, lses, q, rows)


def swa_sink_merge(o_c, lse_c, q, kv_raw, raw_cap, sink, tau, W, positions, rows=None):
    """Merge a compressed-branch result (o_c, lse_c) with the raw-window branch and
    the sink in one normalisation ([cf-1] §3.3):
        M   = max(L_c, L_w, sigma)
        out = (e^{L_c-M} o_c + e^{L_w-M} o_w) / (e^{L_c-M} + e^{L_w-M} + e^{sigma-M})
    where (o_w, L_w) is attention over the window alone without the sink.
    """
    o_c, lse_c, q, kv_raw = _f64(o_c), _f64(lse_c), _f64(q), _f64(kv_raw)
    H = q.shape[2]
    snk = np.full(H, -np.inf) if sink is None else _f64(sink)
    pos = np.asarray(positions)
    pairs = rows if rows is not None else [(b, t) for b in range(q.shape[0]) for t in range(q.shape[1])]
    outs = []
    for n_, (b, t) in enumerate(pairs):
        keys = _window_rows(kv_raw[b], raw_cap, int(pos[b, t]), W) if W > 0 else kv_raw[b, :0]
        o_w, l_w = attend_rows(q[b, t], keys, np.full(H, -np.inf), tau)
        oc = o_c[b, t] if rows is None else o_c[n_]
        lc = lse_c[b, t] if rows is None else lse_c[n_]
        M = np.maximum(np.maximum(lc, l_w), snk)
        M = np.where(np.isfinite(M), M, 0.0)
        ec, ew, es = np.exp(lc - M), np.exp(l_w - M), np.exp(snk - M)
        outs.append((ec[:, None] * oc + ew[:, None] * o_w) / (ec + ew + es)[:, None])
    if rows is None:
        return np.stack(outs).reshape(q.shape)
    return np.stack(outs)


def _reshape_rows(outs, lses, q, rows):
    if rows is None:
        B, T, H, D = q.shape
        return np.stack(outs).reshape(B, T, H, D), np.stack(lses).reshape(B, T, H)
    return np.stack(outs), np.stack(lses)


def round_out(x, dtype: str):
    """Round float64 results once to the output dtype ('f32' or 'bf16')."""
    return formats.bf16(x) if dtype == "bf16" else formats.f32(x)


# ---------------------------------------------------------------------------
# (5) whole layers, composed from the steps above
# ---------------------------------------------------------------------------

def csa_layer(x, m, k, W, tau, dtype, gscale=1.0, rows=None, return_all=False):
    """One CSA layer on host inputs ``x`` (dict of tensors as drawn by the input
    generator): compress KV and indexer keys, NVFP4-quantise indexer q and keys,
    score, select top-k, attend.  ``rows`` restricts scoring/selection/attention
    to a list of (b, t) query rows; compression always covers every token.
    Storage points round once to ``dtype`` ('f32' or 'bf16'); scores to f32 for
    f32 layers and bf16 otherwise.
    """
    q = x["q"]                                  # converted row by row in sparse_attn
    B, T, H, D = q.shape
    pos = np.tile(np.arange(T), (B, 1))
    kv_c = round_out(csa_compress(x["a"], x["b"], x["z"], m), dtype)
    k_src = round_out(csa_compress(x["a_I"], x["b_I"], x["z_I"], m), dtype)
    khat = nvfp4_quantize(k_src, gscale)["xhat"]
    w = x["w"]
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(T)]
    sc_dtype = "f32" if dtype == "f32" else "bf16"
    idx_rows, scores = [], []
    for (b, t) in rows:
        # NVFP4 blocks run along the last dim, so quantising one row is exact
        qh = nvfp4_quantize(_f64(x["q_I"][b:b + 1, t:t + 1]), gscale)["xhat"]
        s = indexer_score(qh, khat[b:b + 1], _f64(w[b:b + 1, t:t + 1]), pos[b:b + 1, t:t + 1], m)
        s = round_scores(s, sc_dtype)
        scores.append(s[0, 0])
        idx_rows.append(topk_select(s, pos[b:b + 1, t:t + 1], m, k)[0, 0])
    idx_rows_by_bt = {(b, t): ir for (b, t), ir in zip(rows, idx_rows)}
    out, lse = sparse_attn(q, kv_c, idx_rows_by_bt, x["kv_raw"], T, x["sink"], tau, W, pos, rows=rows)
    res = {"out": round_out(out, dtype), "lse": formats.f32(lse), "idx": np.stack(idx_rows)}
    if return_all:
        res.update(kv_c=kv_c, k_src=k_src, khat=khat, score=np.stack(scores))
    return res


def hca_layer(x, m, W, tau, dtype, rows=None, return_all=False):
    """One HCA layer: 128:1 compression then dense attention over every visible
    entry plus the raw window and sink.  ``rows`` as in ``csa_layer``."""
    q = x["q"]                                  # converted row by row in dense_attn
    B, T, H, D = q.shape
    pos = np.tile(np.arange(T), (B, 1))
    kv_c = round_out(hca_compress(x["a"], x["z"], m), dtype)
    out, lse = dense_attn(q, kv_c, x["kv_raw"], T, x["sink"], tau, W, pos, m, rows=rows)
    res = {"out": round_out(out, dtype), "lse": formats.f32(lse)}
    if return_all:
        res["kv_c"] = kv_c
    return res


# ---------------------------------------------------------------------------
# Decode (one new token per sequence).  cf-1.com/news/5231315 §3.1/§3.3: the
# compressed cache grows by one entry per m tokens, the raw window keeps the
# last W tokens.  Order of a step at position p: append token p's raw rows to
# the compressor carry (slot p mod 2m); if block (p+1)/m - 1 just completed,
# emit its entry (current block = a rows, predecessor = b rows) into the cache
# before scoring; write token p's raw KV into ring slot p mod W; then score,
# select and attend for the single query, exactly as in prefill.
# ---------------------------------------------------------------------------
def csa_decode_step(st, x, p, m, k, W, tau, dtype, gscale=1.0):
    """One decode step for every sequence at common position ``p``.

    ``st`` (updated in place) holds float64 arrays: ``kv_c`` [B,S,D] and ``khat``
    [B,S,DI] (the cache, S = entries emitted so far), ``ring`` [B,W,D], and the
    carry rings ``carry_<a|b|z|a_I|b_I|z_I>`` [B,2m,dim].  ``x`` holds the step's
    inputs q [B,H,D], q_I [B,HI,DI], w [B,HI], and the new token's a, b, z, a_I,
    b_I, z_I, kv_raw rows.  Returns out [B,H,D] (rounded to ``dtype``), lse
    [B,H], idx [B,k] and the bf16/f32-rounded score [B,S]."""
    for name in ("a", "b", "z", "a_I", "b_I", "z_I"):
        st["carry_" + name][:, p % (2 * m)] = _f64(x[name])
    if (p + 1) % m == 0:
        i = (p + 1) // m - 1
        assert st["kv_c"].shape[1] == i, "cache length must equal the entry being emitted"
        cur = slice((i % 2) * m, (i % 2) * m + m)
        prev = slice(((i + 1) % 2) * m, ((i + 1) % 2) * m + m)

        def entry(a, b, z):
            # entry 0 has no predecessor block: its softmax covers the m current
            # logits only, exactly as in prefill ([cf-1] §3.1 overlap needs a
            # previous block; the first block has none)
            if i == 0:
                cur_rows = [st["carry_" + n][:, cur] for n in (a, b, z)]
                return round_out(csa_compress(cur_rows[0], cur_rows[1], cur_rows[2], m), dtype)
            slab = [np.concatenate([st["carry_" + n][:, prev], st["carry_" + n][:, cur]], axis=1) for n in (a, b, z)]
            return round_out(csa_compress(slab[0], slab[1], slab[2], m, first_has_pred=True), dtype)

        st["kv_c"] = np.concatenate([st["kv_c"], entry("a", "b", "z")], axis=1)
        e_I = entry("a_I", "b_I", "z_I")
        st["khat"] = np.concatenate([st["khat"], nvfp4_quantize(e_I, gscale)["xhat"]], axis=1)
    st["ring"][:, p % W] = _f64(x["kv_raw"])
    q = _f64(x["q"])[:, None]                      # [B,1,H,D]
    B = q.shape[0]
    pos = np.full((B, 1), p, dtype=np.int64)
    qhat = nvfp4_quantize(_f64(x["q_I"])[:, None], gscale)["xhat"]
    sc = indexer_score(qhat, st["khat"], _f64(x["w"])[:, None], pos, m)
    sc = round_scores(sc, "f32" if dtype == "f32" else "bf16")
    idx = topk_select(sc, pos, m, k)
    out, lse = sparse_attn(q, st["kv_c"], idx, st["ring"], W, x["sink"], tau, W, pos)
    return {"out": round_out(out, dtype)[:, 0], "lse": formats.f32(lse)[:, 0], "idx": idx[:, 0],
            "score": sc[:, 0]}


# ---------------------------------------------------------------------------
# (6) grouped output projection ([cf-1] §3.4: with many query heads -- 128 --
# the heads are split into groups, each group's concatenated head outputs are
# projected to a smaller dimension, and the concatenation of the groups is
# projected to the model dimension, which cuts the projection's parameters and
# FLOPs against one projection of all H*D values).
# ---------------------------------------------------------------------------
def grouped_out_proj(o, w1, w2, dtype="bf16"):
    """o [..., H, D] attention output; w1 [g, d_g, (H/g)*D] (group j's
    projection, rows = output features); w2 [d_model, g*d_g].
        y[..., j*d_g:(j+1)*d_g] = o[..., heads of group j, :].flatten() @ w1[j].T
        out = y @ w2.T
    y is rounded once to ``dtype`` (it is stored between the two products), and
    so is the result.  Returns (y, out) as float64 arrays of the rounded values."""
    o, w1, w2 = _f64(o), _f64(w1), _f64(w2)
    g, d_g, kg = w1.shape
    H, D = o.shape[-2], o.shape[-1]
    assert H % g == 0 and kg == (H // g) * D
    lead = o.shape[:-2]
    x = o.reshape(*lead, g, kg)                                    # group j = heads [j H/g, (j+1) H/g)
    y = np.concatenate([x[..., j, :] @ w1[j].T for j in range(g)], axis=-1)
    y = round_out(y, dtype)
    return y, round_out(y @ w2.T, dtype)
