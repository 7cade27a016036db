"""GPU parity of each entry point against the CPU oracle, through the C ABI.

Sizes span several tiles plus ragged tails.  Tolerances:
  * NVFP4 codes/scales and top-k indices: bit-exact;
  * fp32 results: 1e-5 * max(1, |ref|) (the fp32 acceptance bound);
  * bf16 results: the bf16 rounding of the oracle value within one bf16 ulp
    for single-rounding steps (compressors, scores), 2e-2 max-abs for
    attention outputs (the bf16 acceptance bound).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import formats

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def ops(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import ops as o
    return o


def _randn(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(DT[dtype])


def _np(t):
    return t.detach().cpu().to(torch.float64).numpy()


def _ulp_bf16(x):
    """One bf16 ulp at |x| (power-of-two spacing; 2^-133 floor)."""
    x = np.maximum(np.abs(x), 2.0 ** -126)
    _, e = np.frexp(x)
    return np.ldexp(1.0, e - 1 - 7)


def _assert_close(got, ref, dtype):
    if dtype == "f32":
        tol = 1e-5 * np.maximum(1.0, np.abs(ref))
        bad = np.abs(got - ref) > tol
    else:
        bad = np.abs(got - ref) > _ulp_bf16(ref) * 1.0 + 1e-30
    assert not bad.any(), f"{bad.sum()} mismatches; max err {np.abs(got - ref).max():.3e}"


# ------------------------------------------------------------------ NVFP4

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_nvfp4_quantize_bit_exact(ops, dtype):
    rows, D = 1000, 64
    x = _randn((rows, D), dtype, 1) * torch.exp(_randn((rows, 1), "f32", 2) * 3).to(DT[dtype])
    x = x.to(DT[dtype])
    x[0] = 0                                   # all-zero blocks
    x[1, :16] = torch.tensor([6.0, -4, 3, -2, 1.5, -1, 0.5, 0, 5, -5, 2.5, -2.5, 1.25, 0.75, 0.25, 0.1])
    x[2, :16] = 1e-30 if dtype == "f32" else 1e-30   # scale underflows in E4M3
    x[3, :16] = 3e4                            # scale saturates at 448
    for g in (1.0, 0.37):
        xd = x.cuda()
        packed = torch.empty((rows, D // 2), dtype=torch.uint8, device="cuda")
        sf = torch.empty((rows, D // 16), dtype=torch.uint8, device="cuda")
        ops.nvfp4_quantize(xd, packed, sf, gscale=g)
        ref = oracle.nvfp4_quantize(x, g)
        np.testing.assert_array_equal(sf.cpu().numpy(), ref["sf"])
        got = packed.cpu().numpy()
        # +0/-0 codes are the same value; compare canonicalised nibbles and raw bytes
        lo, hi = got & 0xF, got >> 4
        canon = lambda c: np.where(c == 8, 0, c)
        np.testing.assert_array_equal(canon(lo), canon(ref["codes"][:, 0::2]))
        np.testing.assert_array_equal(canon(hi), canon(ref["codes"][:, 1::2]))


def test_e2m1_rounding_every_midpoint_on_gpu(ops):
    """Every E2M1 midpoint and its fp32 neighbours, with scale 1 (amax = 6)."""
    g = formats.E2M1_VALUES
    mids = (g[1:] + g[:-1]) / 2
    vals = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                           np.nextafter(mids.astype(np.float32), np.float32(9)), g]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    n = (len(vals) + 14) // 15 * 15
    pad = np.zeros(n, dtype=np.float32)
    pad[: len(vals)] = vals
    blocks = pad.reshape(-1, 15)
    x = np.concatenate([np.full((blocks.shape[0], 1), 6.0, np.float32), blocks], axis=1)   # amax = 6 -> s = 1
    xt = torch.from_numpy(x).cuda()
    packed = torch.empty((x.shape[0], 8), dtype=torch.uint8, device="cuda")
    sf = torch.empty((x.shape[0], 1), dtype=torch.uint8, device="cuda")
    ops.nvfp4_quantize(xt, packed, sf, 1.0)
    ref = oracle.nvfp4_quantize(x, 1.0)
    got = packed.cpu().numpy()
    codes = np.stack([got & 0xF, got >> 4], -1).reshape(x.shape)
    dec = formats.e2m1_decode(codes) * formats.e4m3_decode(sf.cpu().numpy())
    np.testing.assert_array_equal(dec, ref["xhat"])


# ------------------------------------------------------------- compressors

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,D", [(1, 1030, 64), (2, 517, 128)])
def test_csa_compress(ops, dtype, B, T, D):
    m = 4
    a, b, z = (_randn((B, T, D), dtype, s) for s in (3, 4, 5))
    S = T // m
    out = torch.empty((B, S, D), dtype=DT[dtype], device="cuda")
    fp4 = torch.empty((B, S, D // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((B, S, D // 16), dtype=torch.uint8, device="cuda")
    ops.csa_compress(a.cuda(), b.cuda(), z.cuda(), m, out=out, out_fp4=fp4, out_sf=sf, gscale=1.0)
    ref = oracle.csa_compress(a, b, z, m)
    _assert_close(_np(out), oracle.round_out(ref, dtype) if dtype == "bf16" else ref, dtype)
    # the NVFP4 output is the exact quantisation of the stored entries
    q = oracle.nvfp4_quantize(out.cpu(), 1.0)
    np.testing.assert_array_equal(sf.cpu().numpy(), q["sf"])
    got = fp4.cpu().numpy()
    canon = lambda c: np.where(c == 8, 0, c)
    np.testing.assert_array_equal(canon(got & 0xF), canon(q["codes"][..., 0::2]))
    np.testing.assert_array_equal(canon(got >> 4), canon(q["codes"][..., 1::2]))


def test_csa_compress_decode_window(ops):
    """Decode mode: rings of 2m raw rows, entry emitted only when (p+1) % m == 0."""
    m, D, B = 4, 128, 3
    T = 64
    a, b, z = (_randn((B, T, D), "bf16", s) for s in (6, 7, 8))
    ref = oracle.round_out(oracle.csa_compress(a, b, z, m), "bf16")
    cap = T // m
    out = torch.zeros((B, cap, D), dtype=torch.bfloat16, device="cuda")
    ring = {n: torch.zeros((B, 2 * m, D), dtype=torch.bfloat16, device="cuda") for n in "abz"}
    pos = torch.zeros((B,), dtype=torch.int32, device="cuda")
    src = {"a": a.cuda(), "b": b.cuda(), "z": z.cuda()}
    for p in range(T):
        for n in "abz":
            ops.csa_ring_append(src[n][:, p].contiguous(), ring[n], pos)
        ops.csa_compress(ring["a"], ring["b"], ring["z"], m, out=out, ring_pos=pos, out_bstride=cap)
        ops.csa_pos_advance(pos, 1)
    _assert_close(_np(out), ref, "bf16")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hca_compress(ops, dtype):
    B, T, D, m = 2, 128 * 9 + 50, 128, 128
    a = _randn((B, T, D), dtype, 9)
    z = _randn((B, T, D), dtype, 10, np.sqrt(2.0))
    out = torch.empty((B, T // m, D), dtype=DT[dtype], device="cuda")
    ops.hca_compress(a.cuda(), z.cuda(), m, out)
    ref = oracle.hca_compress(a, z, m)
    _assert_close(_np(out), oracle.round_out(ref, dtype) if dtype == "bf16" else ref, dtype)


# ---------------------------------------------------------------- indexer

def _quant_inputs(ops, B, T, S, HI, DI, seed):
    qi = _randn((B, T, HI, DI), "bf16", seed)
    ki = _randn((B, S, DI), "bf16", seed + 1)
    q4 = torch.empty((B, T, HI, DI // 2), dtype=torch.uint8, device="cuda")
    qs = torch.empty((B, T, HI, DI // 16), dtype=torch.uint8, device="cuda")
    k4 = torch.empty((B, S, DI // 2), dtype=torch.uint8, device="cuda")
    ks = torch.empty((B, S, DI // 16), dtype=torch.uint8, device="cuda")
    ops.nvfp4_quantize(qi.cuda(), q4, qs)
    ops.nvfp4_quantize(ki.cuda(), k4, ks)
    return qi, ki, q4, qs, k4, ks


@pytest.mark.parametrize("HI,DI,sdt", [(4, 64, "bf16"), (2, 32, "f32"), (4, 64, "f32"), (1, 64, "bf16"),
                                       (8, 64, "bf16")])
def test_indexer_score(ops, HI, DI, sdt):
    B, T, m = 2, 700, 4
    S = T // m
    qi, ki, q4, qs, k4, ks = _quant_inputs(ops, B, T, S, HI, DI, 11)
    w = torch.rand((B, T, HI), generator=torch.Generator().manual_seed(3))
    pos0 = torch.tensor([0, 37], dtype=torch.int32)
    score = torch.full((B, T, S), float("nan"), dtype=DT[sdt], device="cuda")
    ops.indexer_score(q4, qs, k4, ks, w.cuda(), pos0.cuda(), score, S, m)
    qhat = oracle.nvfp4_quantize(qi)["xhat"]
    khat = oracle.nvfp4_quantize(ki)["xhat"]
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    ref = oracle.indexer_score(qhat, khat, w, pos, m)
    got = _np(score)
    vis = ~np.isnan(ref)
    assert np.all(~np.isnan(got[vis]))
    if sdt == "f32":
        np.testing.assert_allclose(got[vis], ref[vis], rtol=2e-6, atol=1e-6)
    else:
        _assert_close(got[vis], formats.bf16(ref[vis]), "bf16")
    # the invisible region is left unwritten (still NaN)
    assert np.all(np.isnan(got[~vis]))


def test_indexer_score_row_chunks(ops):
    """Chunked rows (row0 > 0) and a chunk that is not a multiple of the token tile."""
    B, T, S, HI, DI, m = 1, 1000, 250, 4, 64, 4
    qi, ki, q4, qs, k4, ks = _quant_inputs(ops, B, T, S, HI, DI, 21)
    w = torch.rand((B, T, HI), generator=torch.Generator().manual_seed(5)).cuda()
    pos0 = torch.zeros((B,), dtype=torch.int32, device="cuda")
    full = torch.zeros((B, T, S), dtype=torch.float32, device="cuda")
    ops.indexer_score(q4, qs, k4, ks, w, pos0, full, S, m)
    for r0, tc in ((0, 333), (333, 333), (666, 334)):
        part = torch.zeros((B, tc, S), dtype=torch.float32, device="cuda")
        ops.indexer_score(q4, qs, k4, ks, w, pos0, part, S, m, row0=r0, T_chunk=tc)
        torch.testing.assert_close(part, full[:, r0:r0 + tc], rtol=0, atol=0)


@pytest.mark.parametrize("HI", [2, 4, 8])
def test_indexer_score_decode_chunks(ops, HI):
    """Chunks of 1..16/HI query rows take the narrow (N = 16) tile: each chunk
    matches the oracle, with long key rows spanning many entry tiles."""
    B, T, m, DI = 3, 12, 4, 64
    S = 1500
    qi, ki, q4, qs, k4, ks = _quant_inputs(ops, B, T, S, HI, DI, 41)
    w = torch.rand((B, T, HI), generator=torch.Generator().manual_seed(7))
    pos0 = torch.tensor([4 * S - 12, 4 * 700, 4 * S + 40], dtype=torch.int32)
    qhat = oracle.nvfp4_quantize(qi)["xhat"]
    khat = oracle.nvfp4_quantize(ki)["xhat"]
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    ref = oracle.indexer_score(qhat, khat, w, pos, m)
    wd, pd = w.cuda(), pos0.cuda()
    r0 = 0
    for tc in (1, 16 // HI, 1, max(1, 8 // HI), T):
        tc = min(tc, T - r0)
        if tc <= 0:
            break
        part = torch.full((B, tc, S), float("nan"), dtype=torch.float32, device="cuda")
        ops.indexer_score(q4, qs, k4, ks, wd, pd, part, S, m, row0=r0, T_chunk=tc)
        got = _np(part)
        rr = ref[:, r0:r0 + tc]
        vis = ~np.isnan(rr)
        np.testing.assert_allclose(got[vis], rr[vis], rtol=2e-6, atol=1e-6)
        assert np.all(np.isnan(got[~vis]))
        r0 += tc


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("sdt", ["f32", "bf16"])
@pytest.mark.parametrize("k", [1, 7, 64, 512])
def test_topk_bit_exact(ops, sdt, k):
    B, T, m = 2, 600, 4
    S = 9000 // m if k == 512 else T // m
    T = max(T, S * m)
    g = torch.Generator().manual_seed(k)
    sc = torch.randn((B, T, S), generator=g)
    # ties and zeros: quantise a third of the rows coarsely, add +-0
    sc[:, ::3] = torch.round(sc[:, ::3] * 2) / 2
    sc[:, 1::5] = torch.relu(sc[:, 1::5])
    sc[0, 10, :50] = -0.0
    sc = sc.to(DT[sdt])
    pos0 = torch.tensor([0, 3], dtype=torch.int32)
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    ops.topk_select(sc.cuda(), idx, S, m, pos0.cuda())
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    ref = oracle.topk_select(_np(sc), pos, m, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_long_rows_all_equal(ops):
    """A row of identical scores: the k smallest indices."""
    S, k = 20000, 300
    sc = torch.zeros((1, 1, S), dtype=torch.bfloat16, device="cuda")
    pos0 = torch.tensor([4 * S], dtype=torch.int32, device="cuda")
    idx = torch.empty((1, 1, k), dtype=torch.int32, device="cuda")
    ops.topk_select(sc, idx, S, 4, pos0)
    np.testing.assert_array_equal(idx.cpu().numpy()[0, 0], np.arange(k))


@pytest.mark.parametrize("k", [64, 1024, 9000])
def test_topk_multi_cta_rows(ops, k):
    """Few long BF16 rows run split across CTAs through the workspace; the
    result equals the oracle and the one-CTA-per-row path, on repeated calls
    with a workspace that starts out holding garbage."""
    B, T, m, S = 3, 4, 4, 40000
    g = torch.Generator().manual_seed(k + 7)
    sc = torch.randn((B, T, S), generator=g)
    sc[0, 1] = torch.relu(sc[0, 1])                      # many zeros
    sc[1, 0] = torch.round(sc[1, 0] * 4) / 4             # many ties
    sc[1, 2] = 1.5                                       # all equal
    sc[2, 3, ::7] = -0.0
    sc = sc.to(torch.bfloat16)
    pos0 = torch.tensor([4 * S, 4 * 20000 + 1, 4 * 1000], dtype=torch.int32)
    nbytes = ops.topk_workspace_size(B, T, S, k)
    assert nbytes > 0
    ws = torch.full((nbytes // 4,), 12345, dtype=torch.int32, device="cuda")
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    ref = oracle.topk_select(_np(sc), pos, m, k)
    scd, posd = sc.cuda(), pos0.cuda()
    for _ in range(2):
        idx = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
        ops.topk_select(scd, idx, S, m, posd, workspace=ws)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    idx1 = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
    ops.topk_select(scd, idx1, S, m, posd)
    np.testing.assert_array_equal(idx1.cpu().numpy(), ref)


# -------------------------------------------------------------- attention

def _attn_inputs(B, T, H, D, S, dtype, seed, q_scale=1.0):
    q = _randn((B, T, H, D), dtype, seed, q_scale)
    kv_c = _randn((B, S, D), dtype, seed + 1)
    raw = _randn((B, T, D), dtype, seed + 2)
    sink = torch.randn((H,), generator=torch.Generator().manual_seed(seed + 3))
    return q, kv_c, raw, sink


def _attn_tol(dtype):
    return (lambda g, r: np.testing.assert_allclose(g, r, rtol=1e-5, atol=1e-5)) if dtype == "f32" else \
        (lambda g, r: np.testing.assert_allclose(g, r, rtol=0, atol=2e-2))


@pytest.mark.parametrize("dtype,H,D,k", [("f32", 8, 64, 24), ("bf16", 64, 128, 24), ("bf16", 128, 128, 24),
                                         ("bf16", 64, 128, 200), ("bf16", 128, 128, 300)])
def test_sparse_attn(ops, dtype, H, D, k):
    B, T, m, W = 2, 1300, 4, 128
    S = T // m
    tau = 1.0 / np.sqrt(D)
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, dtype, 30)
    pos0 = torch.tensor([0, 5], dtype=torch.int32)
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    idx = oracle.topk_select(np.random.default_rng(0).standard_normal((B, T, S)), pos, m, k)
    idx_t = torch.from_numpy(idx)
    out = torch.empty_like(q, device="cuda")
    lse = torch.empty((B, T, H), dtype=torch.float32, device="cuda")
    ops.sparse_attn_fwd(q.cuda(), kv_c.cuda(), idx_t.cuda(), raw.cuda(), sink.cuda(), tau, W, pos0.cuda(), out,
                        lse)
    ro, rl = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, tau, W, pos)
    _attn_tol(dtype)(_np(out), oracle.round_out(ro, dtype))
    # bf16: the row sums add the bf16-rounded softmax weights (relative error <= 2^-8)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-5 if dtype == "f32" else 0,
                               atol=1e-4 if dtype == "f32" else 2.0 ** -8)


def test_sparse_attn_few_rows_head_split(ops):
    """A call with fewer query rows than SMs and 128 heads runs each row as two
    64-head units: a row chunk [1200, 1240) of two sequences vs the oracle,
    including lse, with rows outside the chunk left untouched."""
    B, T, m, W, H, D, k = 2, 1300, 4, 128, 128, 128, 300
    S = T // m
    tau = 1.0 / np.sqrt(D)
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, "bf16", 31)
    pos0 = torch.tensor([0, 7], dtype=torch.int32)
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    r0, tc = 1200, 40
    idx_full = oracle.topk_select(np.random.default_rng(2).standard_normal((B, T, S)), pos, m, k)
    idx_chunk = torch.from_numpy(np.ascontiguousarray(idx_full[:, r0:r0 + tc]))
    out = torch.zeros((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, T, H), dtype=torch.float32, device="cuda")
    ops.sparse_attn_fwd(q.cuda(), kv_c.cuda(), idx_chunk.cuda(), raw.cuda(), sink.cuda(), tau, W, pos0.cuda(), out,
                        lse, row0=r0, T_chunk=tc)
    rows = [(b, t) for b in range(B) for t in range(r0, r0 + tc)]
    ro, rl = oracle.sparse_attn(q, kv_c, {(b, t): idx_full[b, t] for (b, t) in rows}, raw, T, sink, tau, W, pos,
                                rows=rows)
    got = np.stack([_np(out[b, t]) for (b, t) in rows])
    _attn_tol("bf16")(got, oracle.round_out(ro, "bf16"))
    gl = np.stack([lse[b, t].cpu().numpy() for (b, t) in rows])
    np.testing.assert_allclose(gl, rl, rtol=0, atol=2.0 ** -8)
    assert float(out[:, :r0].abs().max()) == 0.0 and float(out[:, r0 + tc:].abs().max()) == 0.0


@pytest.mark.parametrize("dtype,H,D,m", [("f32", 8, 64, 4), ("bf16", 64, 128, 16), ("bf16", 128, 128, 32),
                                         ("bf16", 16, 128, 4), ("bf16", 32, 128, 128), ("bf16", 64, 128, 128)])
def test_hca_dense_attn(ops, dtype, H, D, m):
    B, T, W = 2, 700, 128
    S = T // m
    tau = 1.0 / np.sqrt(D)
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, dtype, 40)
    pos0 = torch.tensor([0, 9], dtype=torch.int32)
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    out = torch.empty_like(q, device="cuda")
    ops.hca_dense_attn_fwd(q.cuda(), kv_c.cuda(), raw.cuda(), sink.cuda(), tau, W, pos0.cuda(), out, m)
    ro, _ = oracle.dense_attn(q, kv_c, raw, T, sink, tau, W, pos, m)
    _attn_tol(dtype)(_np(out), oracle.round_out(ro, dtype))


@pytest.mark.parametrize("dtype,H,D", [("f32", 16, 64), ("bf16", 64, 128)])
def test_split_path_merge_equals_fused(ops, dtype, H, D):
    """sparse_attn_fwd(W=0, no sink) -> (o_c, lse_c), then swa_sink_merge, equals
    the fused call; both equal the oracle."""
    B, T, m, k, W = 1, 260, 4, 16, 128
    S = T // m
    tau = 0.125
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, dtype, 50)
    pos0 = torch.zeros((B,), dtype=torch.int32)
    pos = np.arange(T)[None]
    idx = oracle.topk_select(np.random.default_rng(1).standard_normal((B, T, S)), pos, m, k)
    dq, dkv, draw, dsink, didx = q.cuda(), kv_c.cuda(), raw.cuda(), sink.cuda(), torch.from_numpy(idx).cuda()
    oc = torch.empty_like(dq)
    lc = torch.empty((B, T, H), dtype=torch.float32, device="cuda")
    ops.sparse_attn_fwd(dq, dkv, didx, draw, None, tau, 0, pos0.cuda(), oc, lc)
    merged = torch.empty_like(dq)
    ops.swa_sink_merge(oc, lc, dq, draw, dsink, tau, W, pos0.cuda(), merged)
    ro, _ = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, tau, W, pos)
    _attn_tol(dtype)(_np(merged), oracle.round_out(ro, dtype))


def test_ring_window_decode_positions(ops):
    """raw_cap < T: the window reads slot j % raw_cap (a decode ring)."""
    B, H, D, cap, W, m = 2, 64, 128, 128, 128, 4
    p0 = np.array([5000, 777])
    S = 2000
    q = _randn((B, 1, H, D), "bf16", 60)
    kv_c = _randn((B, S, D), "bf16", 61)
    ring = _randn((B, cap, D), "bf16", 62)
    sink = torch.randn((H,), generator=torch.Generator().manual_seed(63))
    idx = np.sort(np.random.default_rng(2).choice(S, size=(B, 1, 64), replace=False), axis=-1).astype(np.int32)
    idx[1, 0, 60:] = -1
    out = torch.empty((B, 1, H, D), dtype=torch.bfloat16, device="cuda")
    pos0 = torch.from_numpy(p0.astype(np.int32)).cuda()
    ops.sparse_attn_fwd(q.cuda(), kv_c.cuda(), torch.from_numpy(idx).cuda(), ring.cuda(), sink.cuda(),
                        1 / np.sqrt(D), W, pos0, out, raw_cap=cap)
    ro, _ = oracle.sparse_attn(q, kv_c, idx, ring, cap, sink, 1 / np.sqrt(D), W, p0[:, None])
    _attn_tol("bf16")(_np(out), oracle.round_out(ro, "bf16"))


@pytest.mark.parametrize("H,cap", [(16, 128), (16, 130), (32, 129), (64, 128), (128, 200)])
def test_hca_dense_ring_window(ops, H, cap):
    """Dense (HCA) calls with a raw ring (raw_cap < T): the window reads slot
    j % raw_cap, also when a unit of G = 64/H tokens spans W + G - 1 positions,
    more than the ring holds (the slot wraps more than once within a tile)."""
    B, D, W, m, T = 2, 128, 128, 16, 6
    p0 = np.array([3001, 777])
    S = int(p0.max() + T) // m + 4
    q = _randn((B, T, H, D), "bf16", 80)
    kv_c = _randn((B, S, D), "bf16", 81)
    ring = _randn((B, cap, D), "bf16", 82)
    sink = torch.randn((H,), generator=torch.Generator().manual_seed(83))
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    pos0 = torch.from_numpy(p0.astype(np.int32)).cuda()
    ops.hca_dense_attn_fwd(q.cuda(), kv_c.cuda(), ring.cuda(), sink.cuda(), 1 / np.sqrt(D), W, pos0, out, m,
                           raw_cap=cap)
    pos = p0[:, None] + np.arange(T)[None]
    ro, _ = oracle.dense_attn(q, kv_c, ring, cap, sink, 1 / np.sqrt(D), W, pos, m)
    _attn_tol("bf16")(_np(out), oracle.round_out(ro, "bf16"))


def test_attn_rescale_path(ops):
    """Later KV tiles with far larger logits force the running-max rescale of the
    O^T accumulator and row sums (tiles ordered: entries, then the window)."""
    B, T, H, D, m, k, W = 1, 600, 64, 128, 4, 150, 128
    S = T // m
    q = _randn((B, T, H, D), "bf16", 70, 10.0)         # window logits ~ N(0, 10^2): max ~ 2^5 above
    kv_c = _randn((B, S, D), "bf16", 71, 0.02)          # entries (first tiles): logits ~ 0
    raw = _randn((B, T, D), "bf16", 72)                 # outputs stay O(1)
    sink = torch.randn((H,), generator=torch.Generator().manual_seed(73))
    pos0 = torch.zeros((B,), dtype=torch.int32)
    pos = np.arange(T)[None]
    idx = oracle.topk_select(np.random.default_rng(3).standard_normal((B, T, S)), pos, m, k)
    out = torch.empty_like(q, device="cuda")
    lse = torch.empty((B, T, H), dtype=torch.float32, device="cuda")
    ops.sparse_attn_fwd(q.cuda(), kv_c.cuda(), torch.from_numpy(idx).cuda(), raw.cuda(), sink.cuda(),
                        1 / np.sqrt(D), W, pos0.cuda(), out, lse)
    ro, rl = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, 1 / np.sqrt(D), W, pos)
    _attn_tol("bf16")(_np(out), oracle.round_out(ro, "bf16"))
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=0, atol=2.0 ** -8)


@pytest.mark.parametrize("case", ["sparse_big_logits", "dense_big_logits", "sparse_sink_dominates"])
def test_attn_exact_fallback(ops, case):
    """Units whose softmax arguments leave the fast path's range are recomputed
    exactly: logits far above the sink (clamped arguments), and a sink so large
    that every weight underflows (zero row sums)."""
    B, T, H, D, m, k, W = 1, 400, 64, 128, 4, 48, 128
    S = T // m
    q_scale = 60.0 if "big" in case else 1.0
    q = _randn((B, T, H, D), "bf16", 90, q_scale)
    kv_c = _randn((B, S, D), "bf16", 91)
    raw = _randn((B, T, D), "bf16", 92)
    sink = torch.randn((H,), generator=torch.Generator().manual_seed(93))
    if case == "sparse_sink_dominates":
        sink[::2] = 400.0
    tau = 1 / np.sqrt(D)
    pos0 = torch.zeros((B,), dtype=torch.int32)
    pos = np.arange(T)[None]
    out = torch.empty_like(q, device="cuda")
    lse = torch.empty((B, T, H), dtype=torch.float32, device="cuda")
    if case.startswith("sparse"):
        idx = oracle.topk_select(np.random.default_rng(5).standard_normal((B, T, S)), pos, m, k)
        ops.sparse_attn_fwd(q.cuda(), kv_c.cuda(), torch.from_numpy(idx).cuda(), raw.cuda(), sink.cuda(), tau, W,
                            pos0.cuda(), out, lse)
        ro, rl = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, tau, W, pos)
    else:
        ops.hca_dense_attn_fwd(q.cuda(), kv_c.cuda(), raw.cuda(), sink.cuda(), tau, W, pos0.cuda(), out, m, lse=lse)
        ro, rl = oracle.dense_attn(q, kv_c, raw, T, sink, tau, W, pos, m)
    _attn_tol("bf16")(_np(out), oracle.round_out(ro, "bf16"))
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-5, atol=2.0 ** -8)


def test_attn_row_chunks_and_empty_sets(ops):
    """row0 > 0 chunks write only their rows; W = 0 rows with no entry give 0."""
    B, T, H, D, m, k, W = 1, 700, 64, 128, 4, 64, 128
    S = T // m
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, "bf16", 80)
    pos0 = torch.zeros((B,), dtype=torch.int32, device="cuda")
    pos = np.arange(T)[None]
    idx = oracle.topk_select(np.random.default_rng(4).standard_normal((B, T, S)), pos, m, k)
    dq, dkv, draw, dsink = q.cuda(), kv_c.cuda(), raw.cuda(), sink.cuda()
    full = torch.empty_like(dq)
    ops.sparse_attn_fwd(dq, dkv, torch.from_numpy(idx).cuda(), draw, dsink, 1 / np.sqrt(D), W, pos0, full)
    part = torch.zeros_like(dq)
    for r0, tc in ((0, 250), (250, 250), (500, 200)):
        ops.sparse_attn_fwd(dq, dkv, torch.from_numpy(idx[:, r0:r0 + tc].copy()).cuda(), draw, dsink,
                            1 / np.sqrt(D), W, pos0, part, row0=r0, T_chunk=tc)
    torch.testing.assert_close(part, full, rtol=0, atol=0)
    # no window, no entries for the first m-1 rows: output 0, lse -inf
    o0 = torch.full_like(dq, 7.0)
    l0 = torch.zeros((B, T, H), dtype=torch.float32, device="cuda")
    ops.sparse_attn_fwd(dq, dkv, torch.from_numpy(idx).cuda(), draw, None, 1 / np.sqrt(D), 0, pos0, o0, l0)
    assert torch.all(o0[:, : m - 1] == 0) and torch.all(torch.isinf(l0[:, : m - 1]))
    ro, _ = oracle.sparse_attn(q, kv_c, idx, raw, T, None, 1 / np.sqrt(D), 0, pos)
    _attn_tol("bf16")(_np(o0), oracle.round_out(ro, "bf16"))


def test_attn_unsupported_shapes_rejected(ops):
    q = torch.zeros((1, 8, 16, 64), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 8, 2), dtype=torch.int32, device="cuda")
    pos0 = torch.zeros((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(ops.CsaError):
        ops.sparse_attn_fwd(q, kv, idx, kv, None, 1.0, 0, pos0, torch.empty_like(q))


def test_bounded_wait_timeout_reports_and_recovers(ops):
    """With a 1 ns wait limit the attention kernel's first bounded wait gives
    up: the kernel still returns, the call's own status word reads
    CSA_ERR_TIMEOUT (the library's word stays clear), and with the limit
    restored the same call on the same device gives the oracle's result."""
    B, T, H, D, m, k, W = 1, 160, 64, 128, 4, 16, 128
    S = T // m
    tau = 1.0 / np.sqrt(D)
    q, kv_c, raw, sink = _attn_inputs(B, T, H, D, S, "bf16", 95)
    pos0 = torch.zeros((B,), dtype=torch.int32)
    pos = np.arange(T)[None]
    idx = oracle.topk_select(np.random.default_rng(6).standard_normal((B, T, S)), pos, m, k)
    dq, dkv, draw, dsink, didx = q.cuda(), kv_c.cuda(), raw.cuda(), sink.cuda(), torch.from_numpy(idx).cuda()
    out = torch.zeros_like(dq)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    assert ops.device_status() == 0
    ops.set_wait_timeout_ns(1)
    try:
        ops.sparse_attn_fwd(dq, dkv, didx, draw, dsink, tau, W, pos0.cuda(), out, status=status)
        torch.cuda.synchronize()
    finally:
        ops.set_wait_timeout_ns(0)
    assert int(status.item()) & 0xFF == 5, f"status {int(status.item()):#x}"
    assert ops.device_status() == 0
    status.zero_()
    ops.sparse_attn_fwd(dq, dkv, didx, draw, dsink, tau, W, pos0.cuda(), out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, _ = oracle.sparse_attn(q, kv_c, idx, raw, T, sink, tau, W, pos)
    _attn_tol("bf16")(_np(out), oracle.round_out(ro, "bf16"))


def test_no_device_timeouts(ops):
    torch.cuda.synchronize()
    assert ops.device_status() == 0
