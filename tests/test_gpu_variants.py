"""Variants of the same kernels that the pages name: HCA compression ratio 64
(devpress.csdn.net/awstech/6a462b3a… §3.1, against the 128 of the main
configuration) and top-k 32 / 512 / 1024 (devpress.csdn.net/awstech/6a4623aa…
attention paragraph; cf-1.com/news/5231315 §3.1; yfxerp.com/news/211352 §3).
Same acceptance as the layer tests: index-set overlap and near-tie rule,
outputs within 2e-2 max-abs, against the oracle."""
import pytest

from long_context_compressed_compress_b200 import configs
from test_gpu_layers import L, check_csa, check_hca, sample_rows  # noqa: F401  (fixture re-used)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H", [64, 128])
def test_hca_ratio64(L, H):
    """HCA with 64 tokens per entry: more entries per query, the same window
    and sink; a ragged tail block and two sequences."""
    cfg = configs.scaled(configs.HCA_PREFILL_M64, H=H, T=64 * 45 + 29, seed=21)
    check_hca(L, cfg, sample_rows(cfg.B, cfg.T, 130, 256))


def test_hca_ratio64_full_size_sampled(L):
    """HCA ratio 64 at the full HCA prefill size: B=2, T=131072, 2048 entries."""
    cfg = configs.HCA_PREFILL_M64
    check_hca(L, cfg, sample_rows(cfg.B, cfg.T, 64, 128))


@pytest.mark.parametrize("H,k", [(64, 32), (128, 32), (64, 1024), (128, 512)])
def test_csa_topk_variants(L, H, k):
    """CSA with k = 32 (most rows have many more visible entries than k, so
    the selection is sharp), k = 512 with 128 heads, and k = 1024 with 64 heads
    (rows past 4096 tokens fill the whole top-k set)."""
    cfg = configs.scaled(configs.CSA_PREFILL, H=H, k=k, T=5000, seed=22)
    check_csa(L, cfg, rows=sample_rows(1, cfg.T, 200, 400), chunk=2048)


def test_csa_topk32_full_size_sampled(L):
    """k = 32 at the CSA prefill size (T=32768, 8192 entries)."""
    cfg = configs.CSA_PREFILL_K32
    check_csa(L, cfg, rows=sample_rows(1, cfg.T, 64, 128), chunk=8192)
