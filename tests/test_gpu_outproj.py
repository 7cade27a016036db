"""Grouped output projection (cf-1.com/news/5231315 §3.4) on the tcgen05 GEMM
against the oracle: y (the per-group projections, stored as bf16) and the
final projection, on a ragged row count and at the 128-head size."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import ops
    return ops


def _case(M, H, D, g, d_g, d_model, seed):
    gen = torch.Generator().manual_seed(seed)
    kg = H // g * D
    o = torch.randn((M, H, D), generator=gen).to(torch.bfloat16)
    w1 = (torch.randn((g, d_g, kg), generator=gen) / kg ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((d_model, g * d_g), generator=gen) / (g * d_g) ** 0.5).to(torch.bfloat16)
    return o, w1, w2


def _run(ops, o, w1, w2):
    g, d_g, _ = w1.shape
    y = torch.empty((o.shape[0], g * d_g), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((o.shape[0], w2.shape[0]), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    ops.grouped_out_proj(o.cuda(), w1.cuda(), w2.cuda(), y, out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y.double().cpu().numpy(), out.double().cpu().numpy()


def _absum(o, w1):
    """sum_k |a_k b_k| of every y element: the scale of fp32 accumulation error"""
    g, _, kg = w1.shape
    x = np.abs(o.double().numpy().reshape(o.shape[0], g, kg))
    w = np.abs(w1.double().numpy())
    return np.concatenate([x[:, j] @ w[j].T for j in range(g)], axis=1)


def _check(gy, gout, ry, rout, absum):
    # y: the GPU rounds an fp32 sum, the oracle the exact sum, once each to
    # bf16: one bf16 ulp apart at most, plus the fp32 accumulation error
    # (2^-20 of sum |a b|, which matters only for near-cancelling sums)
    tol = np.abs(ry) * 2.0 ** -7 + 2.0 ** -20 * absum
    assert np.all(np.abs(gy - ry) <= tol), f"y max err {np.abs(gy - ry).max():.3e}"
    assert np.abs(gout - rout).max() <= 2e-2, f"out max err {np.abs(gout - rout).max():.3e}"


@pytest.mark.parametrize("M,H,g,d_g,d_model", [(1000, 128, 8, 256, 512), (300, 64, 4, 512, 256),
                                               (129, 128, 1, 256, 256), (200, 128, 16, 256, 768)])
def test_grouped_out_proj_small(ops, M, H, g, d_g, d_model):
    """Ragged M (TMA rows past the end read zeros, their stores are skipped),
    one group (a plain two-stage projection), many groups."""
    D = 128
    o, w1, w2 = _case(M, H, D, g, d_g, d_model, seed=M + g)
    gy, gout = _run(ops, o, w1, w2)
    ry, rout = oracle.grouped_out_proj(o, w1, w2)
    _check(gy, gout, ry, rout, _absum(o, w1))


def test_grouped_out_proj_full_size_sampled(ops):
    """M = 32768 rows of 128 heads x 128, 8 groups of 16 heads projected to
    1024, model dimension 4096: every GPU row computed, 96 rows checked."""
    M, H, D, g, d_g, d_model = 32768, 128, 128, 8, 1024, 4096
    o, w1, w2 = _case(M, H, D, g, d_g, d_model, seed=7)
    gy, gout = _run(ops, o, w1, w2)
    rows = np.unique(np.concatenate([np.arange(32), np.arange(M - 32, M),
                                     np.random.default_rng(1234).integers(0, M, 32)]))
    ry, rout = oracle.grouped_out_proj(o[rows], w1, w2)
    _check(gy[rows], gout[rows], ry, rout, _absum(o[rows], w1))


def test_grouped_out_proj_rejects_unsupported_shapes(ops):
    o = torch.zeros((4, 128, 128), dtype=torch.bfloat16, device="cuda")
    w1 = torch.zeros((8, 100, 2048), dtype=torch.bfloat16, device="cuda")   # d_g not a multiple of 256
    w2 = torch.zeros((256, 800), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((4, 800), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.CsaError):
        ops.grouped_out_proj(o, w1, w2, y, out)
