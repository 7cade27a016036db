"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, invariants, library routines (torch fp8 casting, torch SDPA in
float64) and brute force on tiny inputs.  Each test is chosen so that a
plausible slip in the oracle (a dropped term, a wrong index or sign, swapped
streams, an off-by-one in visibility or the window) fails it.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from oracle import formats

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- compressors

def _rand(*shape):
    return RNG.standard_normal(shape)


def test_csa_one_hot_gate_selects_single_token_current_block():
    """With one gate logit far above the rest, the entry equals that token's row:
    the ``a`` row when the token is in the current block (an invariant of the definition)."""
    T, D, m = 32, 8, 4
    a, b = _rand(T, D), _rand(T, D)
    for i in range(T // m):
        for j in range(m):
            t = m * i + j
            z = np.full((T, D), -60.0)
            z[t] = 60.0
            e = oracle.csa_compress(a, b, z, m)
            np.testing.assert_array_equal(e[i], a[t])


def test_csa_one_hot_gate_selects_single_token_predecessor_block():
    """...and the ``b`` row when the token is in the predecessor block, so the
    two streams' roles and the overlap offset are pinned."""
    T, D, m = 32, 8, 4
    a, b = _rand(T, D), _rand(T, D)
    for i in range(1, T // m):
        for j in range(m):
            t = m * (i - 1) + j
            z = np.full((T, D), -60.0)
            z[t] = 60.0
            e = oracle.csa_compress(a, b, z, m)
            np.testing.assert_array_equal(e[i], b[t])
            # the same token is the current block of entry i-1 -> a row there
            np.testing.assert_array_equal(e[i - 1], a[t])


def test_csa_constant_gate_is_mean_and_first_entry_masks_predecessor():
    """Constant logits give equal weights: entry i >= 1 is the mean of its 8 rows
    (4 of a, 4 of b); entry 0 is the mean of its 4 a rows (no zero padding)."""
    T, D, m = 40, 6, 4
    a, b = _rand(T, D), _rand(T, D)
    z = np.full((T, D), 5.0)
    e = oracle.csa_compress(a, b, z, m)
    assert e.shape == (T // m, D)
    np.testing.assert_allclose(e[0], a[0:4].mean(0), rtol=1e-14, atol=1e-15)
    for i in range(1, T // m):
        ref = (a[m * i:m * i + m].sum(0) + b[m * i - m:m * i].sum(0)) / (2 * m)
        np.testing.assert_allclose(e[i], ref, rtol=1e-13, atol=1e-15)


def test_csa_trailing_partial_block_emits_nothing_and_decode_window():
    T, D, m = 23, 4, 4
    a, b, z = _rand(T, D), _rand(T, D), _rand(T, D)
    e = oracle.csa_compress(a, b, z, m)
    assert e.shape[0] == 5
    # decode window: rows [4(i-1), 4i+4) with the predecessor present -> entry i
    for i in range(1, 5):
        w = slice(m * (i - 1), m * (i + 1))
        ei = oracle.csa_compress(a[w], b[w], z[w], m, first_has_pred=True)
        assert ei.shape[0] == 1
        np.testing.assert_allclose(ei[0], e[i], rtol=0, atol=0)


def test_csa_two_token_gate_closed_form():
    """Two live logits u, v (rest -inf-like): weights are the logistic pair."""
    T, D, m = 16, 3, 4
    a, b = _rand(T, D), _rand(T, D)
    z = np.full((T, D), -200.0)
    u, v = 0.3, -1.1
    z[6], z[9] = u, v           # entry 2: pred block rows 4..7 (b), current 8..11 (a)
    e = oracle.csa_compress(a, b, z, m)
    wu = 1.0 / (1.0 + np.exp(v - u))
    np.testing.assert_allclose(e[2], wu * b[6] + (1 - wu) * a[9], rtol=1e-13)


def test_hca_special_cases():
    T, D = 512, 5
    a, z = _rand(T, D), _rand(T, D) * np.sqrt(2.0)
    # ratio 1 -> identity
    np.testing.assert_allclose(oracle.hca_compress(a, z, 1), a, rtol=0, atol=0)
    m = 128
    e = oracle.hca_compress(a, z, m)
    assert e.shape == (T // m, D)
    # permutation invariance inside a block
    perm = np.concatenate([RNG.permutation(m) + m * i for i in range(T // m)])
    np.testing.assert_allclose(oracle.hca_compress(a[perm], z[perm], m), e, rtol=1e-13)
    # constant logits -> block mean; one-hot -> that token's row
    np.testing.assert_allclose(oracle.hca_compress(a, np.zeros_like(z), m),
                               a.reshape(T // m, m, D).mean(1), rtol=1e-13, atol=1e-15)
    z1 = np.full((T, D), -80.0)
    z1[m + 17] = 80.0
    np.testing.assert_array_equal(oracle.hca_compress(a, z1, m)[1], a[m + 17])


# ---------------------------------------------------------------------- NVFP4

def test_e4m3_matches_torch_float8_cast():
    """Library special case: torch's float8_e4m3fn cast is RNE; compare on random
    values, every representable value and every midpoint below the overflow edge."""
    vals = formats.e4m3_decode(np.arange(0, 0x7F))
    mids = (vals[1:] + vals[:-1]) / 2
    x32 = np.concatenate([
        vals, mids,
        np.nextafter(mids.astype(np.float32), np.float32(0)).astype(np.float64),
        np.nextafter(mids.astype(np.float32), np.float32(1e9)).astype(np.float64),
        np.abs(RNG.standard_normal(200000)).astype(np.float32) * 3.0,
        np.exp(RNG.uniform(-14, 6, 200000)).astype(np.float32),
    ]).astype(np.float32)
    x32 = x32[x32 <= 464.0]
    ref = torch.from_numpy(x32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = formats.e4m3(x32.astype(np.float64))
    np.testing.assert_array_equal(got, ref)
    # saturation (satfinite): everything above the largest finite value clamps
    assert formats.e4m3(np.array([465.0, 1e6]))[0] == 448.0


def _e2m1_brute(v):
    """Nearest E2M1 value by exhaustive search, ties to the even code."""
    grid = formats.E2M1_VALUES
    out = []
    for x in v:
        mag = min(abs(x), 6.0)
        d = np.abs(grid - mag)
        best = np.flatnonzero(d == d.min())
        pick = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        out.append(np.copysign(grid[pick], x))
    return np.array(out)


def test_e2m1_against_brute_force_including_every_midpoint():
    g = formats.E2M1_VALUES
    mids = (g[1:] + g[:-1]) / 2
    m32 = mids.astype(np.float32)
    cand = np.concatenate([
        g, mids,
        np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(10)),
        RNG.uniform(-8, 8, 20000), [6.5, 7.0, 7.5, 100.0, 0.24, 0.25, 0.26],
    ]).astype(np.float32).astype(np.float64)
    cand = np.concatenate([cand, -cand])
    np.testing.assert_array_equal(formats.e2m1(cand), _e2m1_brute(cand))


def test_fp4_values_are_exact_in_fp8_lossless_dequant():
    """Every E2M1 value is an E4M3 value, so FP4 -> FP8 dequantisation is exact,
    as cf-1.com/news/5231315 §4.4 says (dequantising FP4 to FP8 loses nothing)."""
    g = formats.E2M1_VALUES
    np.testing.assert_array_equal(formats.e4m3(np.concatenate([g, -g])), np.concatenate([g, -g]))


def test_nvfp4_quantize_properties():
    x = RNG.standard_normal((64, 64)).astype(np.float32)
    x[3, :16] = 0.0                                  # all-zero block -> scale 0, codes 0
    r = oracle.nvfp4_quantize(x, 1.0)
    xb = x.reshape(64, 4, 16).astype(np.float64)
    s = r["scale"]
    amax = np.abs(xb).max(-1)
    assert np.all(s[3, 0] == 0) and np.all(r["codes"][3, :16] == 0)
    # the scale is the E4M3 rounding of amax/6 (within one E4M3 step)
    nz = amax > 0
    assert np.all(np.abs(s[nz] - amax[nz] / 6) <= amax[nz] / 6 * 2 ** -4 + 2 ** -10)
    # error bound: |x - xhat| <= half of the local E2M1 spacing (<= 1) times the scale,
    # except values that saturate at 6 * s
    err = np.abs(xb - r["xhat"].reshape(64, 4, 16))
    assert np.all(err <= s[..., None] * 1.0 + 1e-12)
    # codes / packing / scale bytes are consistent with xhat
    deq = formats.e2m1_decode(r["codes"]).reshape(64, 4, 16) * formats.e4m3_decode(r["sf"])[..., None]
    np.testing.assert_array_equal(deq.reshape(64, 64), r["xhat"])
    lo, hi = r["packed"] & 0xF, r["packed"] >> 4
    np.testing.assert_array_equal(lo, r["codes"][:, 0::2])
    np.testing.assert_array_equal(hi, r["codes"][:, 1::2])
    # values already on the grid round-trip exactly (scale 1: amax = 6)
    y = np.tile(np.array([6.0, -4, 3, -2, 1.5, -1, 0.5, 0] * 2, dtype=np.float32), (2, 1))
    np.testing.assert_array_equal(oracle.nvfp4_quantize(y, 1.0)["xhat"], y.astype(np.float64))


def test_nvfp4_global_scale():
    x = RNG.standard_normal((8, 32)).astype(np.float32) * 2000.0
    r1 = oracle.nvfp4_quantize(x, 1.0)
    # with g = 1 the scale of a block with amax ~6000 saturates at 448
    assert r1["scale"].max() == 448.0
    # ...so values beyond 6*448 clamp and break the half-spacing error bound
    def within_bound(r, g):
        s = r["scale"][..., None] * np.float64(np.float32(g))
        err = np.abs(r["xhat"].reshape(8, 2, 16) - x.reshape(8, 2, 16).astype(np.float64))
        return np.all(err <= s * 1.0 + 1e-9)
    assert not within_bound(r1, 1.0)
    # a global scale g = amax / (6 * 448) keeps every block scale finite: bound holds
    g = float(np.abs(x).max() / (6 * 448))
    r2 = oracle.nvfp4_quantize(x, g)
    assert r2["scale"].max() <= 448.0
    assert within_bound(r2, g)


# -------------------------------------------------------------------- indexer

def _indexer_brute(qh, kh, w, pos, m):
    B, T, H, C = qh.shape
    S = kh.shape[1]
    out = np.full((B, T, S), np.nan)
    for b, t, s in itertools.product(range(B), range(T), range(S)):
        if m * (s + 1) - 1 > pos[b, t]:
            continue
        acc = 0.0
        for h in range(H):
            d = 0.0
            for c in range(C):
                d += qh[b, t, h, c] * kh[b, s, c]
            acc += w[b, t, h] * max(d, 0.0)
        out[b, t, s] = acc
    return out


def test_indexer_matches_brute_force_loops():
    B, T, H, C, m = 2, 13, 3, 5, 4
    S = T // m
    qh, kh, w = _rand(B, T, H, C), _rand(B, S, C), RNG.uniform(0, 1, (B, T, H))
    pos = np.tile(np.arange(T), (B, 1)) + np.array([[0], [5]])
    got = oracle.indexer_score(qh, kh, w, pos, m)
    ref = _indexer_brute(qh, kh, w, pos, m)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_allclose(got[~np.isnan(got)], ref[~np.isnan(ref)], rtol=1e-12, atol=1e-14)
    # visibility: position p sees exactly (p+1)//m entries
    assert np.all((~np.isnan(got)).sum(-1) == np.minimum((pos + 1) // m, S))


def test_indexer_relu_and_head_weights():
    B, T, H, C, m = 1, 8, 2, 4, 1
    qh, kh = _rand(B, T, H, C), _rand(B, T, C)
    w = np.zeros((B, T, H))
    w[..., 1] = 1.0
    pos = np.arange(T)[None]
    got = oracle.indexer_score(qh, kh, w, pos, m)
    dots = qh[0, :, 1, :] @ kh[0].T
    ref = np.where(np.tril(np.ones((T, T))) > 0, np.maximum(dots, 0), np.nan)
    np.testing.assert_allclose(got[0], ref, rtol=1e-13, atol=0)
    assert np.nanmin(got) >= 0.0


# ---------------------------------------------------------------------- top-k

def _topk_brute(row, n, k):
    cand = sorted(range(n), key=lambda s: (-(row[s] + 0.0), s))[:k]
    return sorted(cand)


def test_topk_matches_brute_force_sort_with_ties_and_zeros():
    m, k = 4, 5
    T = 64
    S = T // m
    pos = np.arange(T)[None]
    for trial in range(6):
        # few distinct values -> many ties; include +0 and -0
        vals = np.array([0.0, -0.0, 1.0, 2.0, 0.5, -1.0])
        sc = RNG.choice(vals, size=(1, T, S)) if trial % 2 == 0 else np.round(RNG.standard_normal((1, T, S)), 1)
        got = oracle.topk_select(sc, pos, m, k)
        for t in range(T):
            n = min((t + 1) // m, S)
            ref = _topk_brute(sc[0, t], n, k)
            exp = np.full(k, -1)
            exp[: len(ref)] = ref
            np.testing.assert_array_equal(got[0, t], exp)


def test_topk_k_at_least_visible_returns_all_visible():
    m, T, k = 4, 40, 64
    sc = RNG.standard_normal((1, T, T // m))
    got = oracle.topk_select(sc, np.arange(T)[None], m, k)
    for t in range(T):
        n = (t + 1) // m
        np.testing.assert_array_equal(got[0, t, :n], np.arange(n))
        assert np.all(got[0, t, n:] == -1)


# ------------------------------------------------------------------ attention

def _sdpa(q, k, v, scale, mask=None, causal=False):
    qt = torch.from_numpy(q).transpose(1, 2)      # [B,H,T,D]
    kt = torch.from_numpy(k)[:, None]             # [B,1,T,D]
    vt = torch.from_numpy(v)[:, None]
    H = qt.shape[1]
    kt, vt = kt.expand(-1, H, -1, -1), vt.expand(-1, H, -1, -1)
    am = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, is_causal=causal, scale=scale)
    return o.transpose(1, 2).numpy()


def test_hca_ratio_one_no_window_no_sink_equals_causal_sdpa():
    """Invariant: HCA with ratio 1 is causal dense attention."""
    B, T, H, D, tau = 2, 37, 3, 8, 0.3
    q, x = _rand(B, T, H, D), _rand(B, T, D)
    e = oracle.hca_compress(x, _rand(B, T, D), 1)          # ratio 1: e == x
    pos = np.tile(np.arange(T), (B, 1))
    out, _ = oracle.dense_attn(q, e, x, T, None, tau, 0, pos, 1)
    np.testing.assert_allclose(out, _sdpa(q, x, x, tau, causal=True), rtol=1e-12, atol=1e-13)


def test_window_only_equals_banded_sdpa():
    """The raw window is j in (p - W, p]: attention with k = 0 entries and W = 5
    equals SDPA under a banded mask (pins the window bounds)."""
    B, T, H, D, W, tau = 1, 30, 2, 6, 5, 0.7
    q, x = _rand(B, T, H, D), _rand(B, T, D)
    kv_c = np.zeros((B, 1, D))
    idx = np.full((B, T, 3), -1, dtype=np.int32)
    pos = np.arange(T)[None]
    out, _ = oracle.sparse_attn(q, kv_c, idx, x, T, None, tau, W, pos)
    i, j = np.arange(T)[:, None], np.arange(T)[None, :]
    band = (j <= i) & (j > i - W)
    mask = np.where(band, 0.0, -np.inf)
    np.testing.assert_allclose(out, _sdpa(q, x, x, tau, mask=mask), rtol=1e-12, atol=1e-13)


def test_csa_with_k_covering_all_entries_equals_dense():
    """Invariant: with k >= S, CSA equals dense attention over entries."""
    B, T, H, D, m, W = 1, 64, 4, 8, 4, 7
    S = T // m
    q, kv_c, raw = _rand(B, T, H, D), _rand(B, S, D), _rand(B, T, D)
    sink = _rand(H)
    pos = np.arange(T)[None]
    sc = RNG.standard_normal((B, T, S))
    idx = oracle.topk_select(sc, pos, m, S + 3)
    o1, l1 = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, 0.4, W, pos)
    o2, l2 = oracle.dense_attn(q, kv_c, raw, T, sink, 0.4, W, pos, m)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


def test_sink_closed_form_only_lowers_mass():
    """out_sigma = out_nosink * Z / (Z + e^sigma), Z = e^lse (the sink
    only lowers attention mass)."""
    B, T, H, D, m, W = 1, 48, 5, 8, 4, 16
    S = T // m
    q, kv_c, raw = _rand(B, T, H, D), _rand(B, S, D), _rand(B, T, D)
    sink = RNG.standard_normal(H) * 2
    pos = np.arange(T)[None]
    o0, l0 = oracle.dense_attn(q, kv_c, raw, T, None, 0.5, W, pos, m)
    o1, l1 = oracle.dense_attn(q, kv_c, raw, T, sink, 0.5, W, pos, m)
    Z = np.exp(l0)
    np.testing.assert_allclose(o1, o0 * (Z / (Z + np.exp(sink)))[..., None], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l0, l1)
    assert np.all(np.abs(o1) <= np.abs(o0) + 1e-15)


def test_merge_split_path_equals_fused_path():
    B, T, H, D, m, W, k = 2, 40, 3, 8, 4, 9, 4
    S = T // m
    q, kv_c, raw = _rand(B, T, H, D), _rand(B, S, D), _rand(B, T, D)
    sink = _rand(H)
    pos = np.tile(np.arange(T), (B, 1)) + np.array([[0], [3]])
    idx = oracle.topk_select(RNG.standard_normal((B, T, S)), pos, m, k)
    raw_cap = T + 3
    raw_full = _rand(B, raw_cap, D)
    fused, _ = oracle.sparse_attn(q, kv_c, idx, raw_full, raw_cap, sink, 0.6, W, pos)
    oc, lc = oracle.sparse_attn(q, kv_c, idx, raw_full, raw_cap, None, 0.6, 0, pos)
    split = oracle.swa_sink_merge(oc, lc, q, raw_full, raw_cap, sink, 0.6, W, pos)
    np.testing.assert_allclose(split, fused, rtol=1e-12, atol=1e-14)


def test_ring_buffer_slots_equal_linear_history():
    """Raw token j lives at slot j % raw_cap: a 16-slot ring holding the last 16
    tokens gives the same window as the full linear history (W <= cap)."""
    B, T, H, D, W, cap = 1, 50, 2, 4, 16, 16
    q, raw = _rand(B, T, H, D), _rand(B, T, D)
    pos = np.arange(T)[None]
    t = T - 1
    ring = np.zeros((B, cap, D))
    for j in range(T - cap, T):
        ring[0, j % cap] = raw[0, j]
    idx = np.full((B, T, 1), -1, dtype=np.int32)
    kv_c = np.zeros((B, 1, D))
    o_lin, _ = oracle.sparse_attn(q, kv_c, idx, raw, T, None, 1.0, W, pos, rows=[(0, t)])
    o_ring, _ = oracle.sparse_attn(q, kv_c, idx, ring, cap, None, 1.0, W, pos, rows=[(0, t)])
    np.testing.assert_array_equal(o_lin, o_ring)


def test_bf16_rounding_matches_torch_on_fp32_inputs():
    """For fp32-representable inputs a single RNE to bf16 is what torch's cast does."""
    x = (RNG.standard_normal(100000) * np.exp(RNG.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(formats.bf16(x.astype(np.float64)), ref)


def _decode_from(T0, T=96, W=16):
    """Decode tokens T0..T-1 from a cache built from tokens [0, T0) and return
    (per-step results, full prefill oracle result, final state)."""
    from long_context_compressed_compress_b200 import configs, inputs
    cfg = configs.scaled(configs.PR1, T=T, k=8)
    m = cfg.m
    x = inputs.layer_inputs(cfg, device="cpu")
    full = oracle.csa_layer(x, m, cfg.k, W, cfg.tau, cfg.dtype)
    f = {k: v.to(torch.float64).numpy() for k, v in x.items()}
    st = {"kv_c": oracle.round_out(oracle.csa_compress(f["a"][:, :T0], f["b"][:, :T0], f["z"][:, :T0], m), "f32"),
          "ring": np.zeros((cfg.B, W, cfg.D))}
    k_src = oracle.round_out(oracle.csa_compress(f["a_I"][:, :T0], f["b_I"][:, :T0], f["z_I"][:, :T0], m), "f32")
    st["khat"] = oracle.nvfp4_quantize(k_src)["xhat"] if k_src.shape[1] else np.zeros((cfg.B, 0, cfg.DI))
    for j in range(max(0, T0 - W), T0):
        st["ring"][:, j % W] = f["kv_raw"][:, j]
    # the carry holds the raw rows of the last complete block and of the
    # block in progress
    for n in ("a", "b", "z", "a_I", "b_I", "z_I"):
        c = np.zeros((cfg.B, 2 * m, f[n].shape[-1]))
        for j in range(max(0, (T0 // m - 1) * m), T0):
            c[:, j % (2 * m)] = f[n][:, j]
        st["carry_" + n] = c
    res = []
    for p in range(T0, cfg.T):
        xs = {n: f[n][:, p] for n in ("q", "q_I", "w", "a", "b", "z", "a_I", "b_I", "z_I", "kv_raw")}
        xs["sink"] = f["sink"]
        res.append(oracle.csa_decode_step(st, xs, p, m, cfg.k, W, cfg.tau, cfg.dtype))
    return res, full, st, cfg


@pytest.mark.parametrize("T0", [64, 0, 1, 3, 5])
def test_decode_steps_equal_prefill_rows(T0):
    """Decoding token p from a cache built from tokens [0, T0) gives row p of a
    prefill over the same tokens: pins the decode step's carry slots, emission
    timing (entry (p+1)/m - 1 visible at step p), entry 0 without a predecessor
    (T0 < m: the first block's softmax covers its own m logits only), NVFP4
    keys and the ring window."""
    res, full, st, cfg = _decode_from(T0)
    for p, r in zip(range(T0, cfg.T), res):
        np.testing.assert_array_equal(r["idx"][0], full["idx"][p])     # rows are (b, t), B = 1
        np.testing.assert_allclose(r["out"][0], full["out"][p], rtol=1e-12, atol=1e-12)
    assert st["kv_c"].shape[1] == cfg.T // cfg.m
    # the emitted cache itself equals the prefill compressor's entries, entry 0
    # included (a planted predecessor at entry 0 changes it: see the next test)
    from long_context_compressed_compress_b200 import inputs
    x = inputs.layer_inputs(cfg, device="cpu")
    ref = oracle.round_out(oracle.csa_compress(x["a"], x["b"], x["z"], cfg.m), "f32")
    np.testing.assert_array_equal(st["kv_c"], ref)


def test_decode_entry0_differs_from_a_zero_predecessor():
    """Entry 0 with a zero predecessor slab (8 logits, four of them 0) is not
    entry 0 of the definition; the decode step must emit the latter."""
    res, full, st, cfg = _decode_from(0, T=8)
    f = {}
    from long_context_compressed_compress_b200 import inputs
    x = inputs.layer_inputs(cfg, device="cpu")
    m = cfg.m
    slab = [np.concatenate([np.zeros((1, m, cfg.D)), x[n][:, :m].double().numpy()], axis=1) for n in ("a", "b", "z")]
    wrong = oracle.round_out(oracle.csa_compress(slab[0], slab[1], slab[2], m, first_has_pred=True), "f32")
    assert np.abs(wrong[:, 0] - st["kv_c"][:, 0]).max() > 1e-3


# ------------------------------------------------------- grouped out projection

def test_grouped_out_proj_one_group_is_the_plain_two_stage_projection():
    """g = 1: y = o.flatten() @ w1[0].T, out = y @ w2.T (torch matmul, fp64)."""
    o = RNG.standard_normal((5, 4, 8))
    w1 = RNG.standard_normal((1, 6, 32))
    w2 = RNG.standard_normal((7, 6))
    y, out = oracle.grouped_out_proj(o, w1, w2, dtype="f32")
    yt = torch.from_numpy(o.reshape(5, 32)) @ torch.from_numpy(w1[0]).T
    np.testing.assert_allclose(y, formats.f32(yt.numpy()), rtol=1e-6)
    np.testing.assert_allclose(out, formats.f32((torch.from_numpy(y) @ torch.from_numpy(w2).T).numpy()),
                               rtol=1e-6)


def test_grouped_out_proj_identity_groups_reduce_to_one_projection():
    """Each w1 block the identity (d_g = (H/g) D): the result is the ungrouped
    output projection o.flatten() @ w2.T, i.e. the grouping only regroups."""
    T, H, D, g = 6, 8, 4, 4
    o = RNG.standard_normal((T, H, D))
    kg = H // g * D
    w1 = np.stack([np.eye(kg) for _ in range(g)])
    w2 = RNG.standard_normal((5, g * kg))
    _, out = oracle.grouped_out_proj(o, w1, w2, dtype="f32")
    ref = (torch.from_numpy(o.reshape(T, H * D)) @ torch.from_numpy(w2).T).numpy()
    # y is stored (rounded to fp32) between the products: the gap is within
    # fp32 rounding of the 32-term sums
    np.testing.assert_allclose(out, formats.f32(ref), rtol=1e-5, atol=1e-5)


def test_grouped_out_proj_groups_follow_head_order():
    """Group j is heads [j H/g, (j+1) H/g): zeroing group 1's heads in o zeroes
    exactly group 1's slice of y; permuting the groups (heads, w1 blocks and
    w2 column blocks together) leaves the result unchanged."""
    T, H, D, g, dg = 3, 8, 2, 4, 3
    o = RNG.standard_normal((T, H, D))
    w1 = RNG.standard_normal((g, dg, H // g * D))
    w2 = RNG.standard_normal((4, g * dg))
    o0 = o.copy()
    o0[:, 2:4] = 0.0
    y0, _ = oracle.grouped_out_proj(o0, w1, w2, dtype="f32")
    assert np.all(y0[:, dg:2 * dg] == 0) and np.all(y0[:, :dg] != 0)
    perm = [2, 0, 3, 1]
    op = np.concatenate([o[:, 2 * j:2 * j + 2] for j in perm], axis=1)
    w2p = np.concatenate([w2[:, dg * j:dg * j + dg] for j in perm], axis=1)
    _, out = oracle.grouped_out_proj(o, w1, w2, dtype="f32")
    _, outp = oracle.grouped_out_proj(op, w1[perm], w2p, dtype="f32")
    np.testing.assert_allclose(outp, out, rtol=1e-6, atol=1e-9)
