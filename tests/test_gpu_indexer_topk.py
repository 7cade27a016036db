"""GPU parity of the fused indexer -> top-k kernel (indexer_topk) through the
C ABI.

  * exact-grid inputs: NVFP4 codes on the E2M1 grid with unit block scales and
    head weights that are multiples of 1/8, so every score is an exact fp32
    value on both sides and its BF16 rounding is the oracle's: the selected
    indices must equal oracle.topk_select on the oracle's BF16 scores bit for
    bit (integer-valued scores make ties common; rows whose k-th key lies more
    than the selection window below the row maximum are present and checked);
  * random inputs: the fused result equals indexer_score + topk_select bit for
    bit, and against the oracle every disagreement is a near-tie;
  * edge cases: rows with fewer visible entries than k, empty rows, row chunks,
    all-equal rows, negative weights, the full prefill size.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import formats

pytestmark = pytest.mark.gpu

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(scope="module")
def ops(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import ops as o
    return o


def _grid_values(shape, rng):
    """Values on the E2M1 grid, each 16-block holding one +-6 (block scale 1)."""
    v = rng.choice(GRID, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    blocks = v.reshape(-1, 16)
    pos = rng.integers(0, 16, size=blocks.shape[0])
    blocks[np.arange(blocks.shape[0]), pos] = 6.0 * rng.choice([-1.0, 1.0], size=blocks.shape[0])
    return blocks.reshape(shape)


def _quantise(ops, x):
    xt = torch.from_numpy(x).to(torch.bfloat16).cuda()
    packed = torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device="cuda")
    sf = torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=torch.uint8, device="cuda")
    ops.nvfp4_quantize(xt, packed, sf)
    return packed, sf


def _grid_case(ops, B, T, S, HI, seed, w_lo=-1.0, w_hi=2.0):
    rng = np.random.default_rng(seed)
    q = _grid_values((B, T, HI, 64), rng)
    kx = _grid_values((B, S, 64), rng)
    w = rng.integers(int(w_lo * 8), int(w_hi * 8), size=(B, T, HI)) / 8.0
    # the quantisation is exact on these inputs (oracle side)
    assert np.array_equal(oracle.nvfp4_quantize(q)["xhat"], q)
    assert np.array_equal(oracle.nvfp4_quantize(kx)["xhat"], kx)
    q4, qs = _quantise(ops, q)
    k4, ks = _quantise(ops, kx)
    return q, kx, w, q4, qs, k4, ks


def _keys(v):
    """Order-preserving 16-bit keys of BF16 values (+0 == -0)."""
    b = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    u = b.astype(np.int64) & 0xFFFF
    u = np.where(u == 0x8000, 0, u)
    return np.where(u & 0x8000, (~u) & 0xFFFF, u | 0x8000)


def _run(ops, q4, qs, k4, ks, w, pos0, S, m, k, row0=0, T_chunk=None):
    B, T = q4.shape[0], q4.shape[1]
    tc = T - row0 if T_chunk is None else T_chunk
    idx = torch.full((B, tc, k), -7, dtype=torch.int32, device="cuda")
    ops.indexer_topk(q4, qs, k4, ks, torch.from_numpy(w).float().cuda(), torch.from_numpy(pos0).cuda(), idx, S, m,
                     row0=row0, T_chunk=tc)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("HI,k", [(4, 16), (4, 100), (4, 512), (8, 64), (8, 300)])
def test_exact_grid_bit_exact_vs_oracle(ops, HI, k):
    B, T, m = 2, 2900, 4
    S = T // m                                   # 725: two full chunks and a ragged third
    q, kx, w, q4, qs, k4, ks = _grid_case(ops, B, T, S, HI, 100 + k + HI)
    pos0 = np.array([0, 37], dtype=np.int32)
    pos = np.arange(T)[None] + pos0[:, None]
    ref_sc = oracle.round_scores(oracle.indexer_score(q, kx, w, pos, m), "bf16")
    ref = oracle.topk_select(ref_sc, pos, m, k)
    got = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k)
    np.testing.assert_array_equal(got, ref)
    # the inputs reach the window's fallback: some row's k-th key lies more than
    # 1024 keys below its maximum
    far = 0
    vis = oracle.visible_entries(pos, m)
    for b in range(B):
        for t in range(0, T, 7):
            n = int(min(vis[b, t], S))
            if n > k:
                kk = np.sort(_keys(ref_sc[b, t, :n]))[::-1]
                far += int(kk[0] - kk[k - 1] >= 1024)
    assert far > 0


def test_row_chunks_and_positions(ops):
    """Chunks of rows (row0 > 0, ragged T_chunk) at per-sequence positions,
    against one call over all rows and against the oracle."""
    B, T, m, HI, k = 3, 1500, 4, 4, 64
    S = 600
    q, kx, w, q4, qs, k4, ks = _grid_case(ops, B, T, S, HI, 7)
    pos0 = np.array([0, 4 * 300 + 2, 4 * S], dtype=np.int32)
    pos = np.arange(T)[None] + pos0[:, None]
    ref = oracle.topk_select(oracle.round_scores(oracle.indexer_score(q, kx, w, pos, m), "bf16"), pos, m, k)
    full = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k)
    np.testing.assert_array_equal(full, ref)
    r0 = 0
    for tc in (1, 7, 333, 1159):
        part = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k, row0=r0, T_chunk=tc)
        np.testing.assert_array_equal(part, ref[:, r0:r0 + tc])
        r0 += tc


def test_all_equal_and_negative_rows(ops):
    """Zero weights make every score +0 (the k smallest indices); negative
    weights make every score <= 0."""
    B, T, m, HI, k = 2, 1200, 4, 4, 40
    S = T // m
    q, kx, w, q4, qs, k4, ks = _grid_case(ops, B, T, S, HI, 9)
    w[0] = 0.0
    w[1] = -np.abs(w[1]) - 0.125
    pos0 = np.zeros((B,), dtype=np.int32)
    pos = np.arange(T)[None] + pos0[:, None]
    ref_sc = oracle.round_scores(oracle.indexer_score(q, kx, w, pos, m), "bf16")
    ref = oracle.topk_select(ref_sc, pos, m, k)
    got = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k)
    np.testing.assert_array_equal(got, ref)
    n_last = min(S, T // m)
    np.testing.assert_array_equal(got[0, -1], np.arange(k))
    assert n_last > k


def test_empty_and_short_rows(ops):
    """Rows that see no entry get -1 everywhere; rows that see fewer than k get
    0 .. n-1 then -1; a sequence with S = 0 entries."""
    B, T, m, HI, k = 1, 64, 4, 4, 32
    S = 16
    q, kx, w, q4, qs, k4, ks = _grid_case(ops, B, T, S, HI, 11)
    pos0 = np.zeros((B,), dtype=np.int32)
    got = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k)
    for t in range(T):
        n = min(S, (t + 1) // m)
        np.testing.assert_array_equal(got[0, t], np.concatenate([np.arange(n), -np.ones(k - n)]).astype(np.int32))
    got0 = _run(ops, q4, qs, k4, ks, w, pos0, 0, m, k)
    assert np.all(got0 == -1)


def _random_case(ops, B, T, S, HI, seed):
    g = torch.Generator().manual_seed(seed)
    qi = torch.randn((B, T, HI, 64), generator=g).to(torch.bfloat16)
    ki = torch.randn((B, S, 64), generator=g).to(torch.bfloat16)
    w = torch.rand((B, T, HI), generator=g).numpy().astype(np.float32)
    q4 = torch.empty((B, T, HI, 32), dtype=torch.uint8, device="cuda")
    qs = torch.empty((B, T, HI, 4), dtype=torch.uint8, device="cuda")
    k4 = torch.empty((B, S, 32), dtype=torch.uint8, device="cuda")
    ks = torch.empty((B, S, 4), dtype=torch.uint8, device="cuda")
    ops.nvfp4_quantize(qi.cuda(), q4, qs)
    ops.nvfp4_quantize(ki.cuda(), k4, ks)
    return qi, ki, w, q4, qs, k4, ks


def _unfused(ops, q4, qs, k4, ks, w, pos0, S, m, k):
    B, T = q4.shape[0], q4.shape[1]
    score = torch.empty((B, T, S), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    wd, pd = torch.from_numpy(w).cuda(), torch.from_numpy(pos0).cuda()
    ops.indexer_score(q4, qs, k4, ks, wd, pd, score, S, m)
    ops.topk_select(score, idx, S, m, pd)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def _near_tie_check(got, ref_idx, ref_sc, rows):
    bad = 0
    for (b, t) in rows:
        ro = set(ref_idx[b, t][ref_idx[b, t] >= 0].tolist())
        go = set(got[b, t][got[b, t] >= 0].tolist())
        if ro == go:
            continue
        sc = ref_sc[b, t]
        kth = np.sort(sc[list(ro)])[0]
        ulp = 2 * formats.bf16(np.abs(kth)) * 2.0 ** -8
        bad += sum(abs(sc[s] - kth) > ulp + 1e-30 for s in ro ^ go)
    assert bad == 0, f"{bad} disagreements that are not near-ties"


@pytest.mark.parametrize("HI", [4, 8])
def test_random_equals_unfused_and_oracle(ops, HI):
    B, T, m, k = 2, 4100, 4, 512
    S = T // m
    qi, ki, w, q4, qs, k4, ks = _random_case(ops, B, T, S, HI, 31 + HI)
    pos0 = np.array([0, 5], dtype=np.int32)
    got = _run(ops, q4, qs, k4, ks, w, pos0, S, m, k)
    np.testing.assert_array_equal(got, _unfused(ops, q4, qs, k4, ks, w, pos0, S, m, k))
    pos = np.arange(T)[None] + pos0[:, None]
    qhat = oracle.nvfp4_quantize(qi)["xhat"]
    khat = oracle.nvfp4_quantize(ki)["xhat"]
    ref_sc = oracle.indexer_score(qhat, khat, w, pos, m)
    ref = oracle.topk_select(oracle.round_scores(ref_sc, "bf16"), pos, m, k)
    rows = [(b, t) for b in range(B) for t in range(0, T, 3)]
    _near_tie_check(got, ref, ref_sc, rows)


def test_full_prefill_size(ops):
    """The CSA prefill shape (T = 32768, S = 8192, k = 512): equal to the
    unfused path on every row, near-ties only against the oracle on a sample."""
    from long_context_compressed_compress_b200 import configs
    c = configs.CSA_PREFILL
    assert c.S <= ops.indexer_topk_max_entries(c.HI, c.DI)
    qi, ki, w, q4, qs, k4, ks = _random_case(ops, c.B, c.T, c.S, c.HI, 77)
    pos0 = np.zeros((c.B,), dtype=np.int32)
    got = _run(ops, q4, qs, k4, ks, w, pos0, c.S, c.m, c.k)
    np.testing.assert_array_equal(got, _unfused(ops, q4, qs, k4, ks, w, pos0, c.S, c.m, c.k))
    rng = np.random.default_rng(1234)
    ts = sorted(set(range(0, 64)) | set(range(c.T - 64, c.T)) | set(rng.integers(0, c.T, 64).tolist()))
    pos = np.arange(c.T)[None]
    qhat = oracle.nvfp4_quantize(qi[:, ts])["xhat"]
    khat = oracle.nvfp4_quantize(ki)["xhat"]
    ref_sc = oracle.indexer_score(qhat, khat, w[:, ts], pos[:, ts], c.m)
    ref = oracle.topk_select(oracle.round_scores(ref_sc, "bf16"), pos[:, ts], c.m, c.k)
    _near_tie_check(got[:, ts], ref, ref_sc, [(0, i) for i in range(len(ts))])
