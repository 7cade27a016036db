"""topk_select_noalloc (the library's fixed scratch instead of a caller
workspace) against topk_select with a workspace, on two calls in a row.  Kept
in its own file, collected last, and independent of the other tests' state."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import ops
    return ops


def _case(seed, B, T, S):
    g = torch.Generator().manual_seed(seed)
    sc = torch.randn((B, T, S), generator=g)
    sc[0, 0] = torch.relu(sc[0, 0])                  # ties at zero
    sc[-1, -1] = torch.round(sc[-1, -1] * 4) / 4     # many ties
    return sc.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,T,S,k", [(4, 2, 40000, 1024), (32, 1, 262161, 1024), (2, 3, 20000, 77)])
def test_noalloc_equals_workspace_path_twice(ops, B, T, S, k):
    m = 4
    assert 0 < ops.topk_workspace_size(B, T, S, k) <= 1 << 20
    pos0 = torch.tensor([4 * S - 3 * (b % 3) for b in range(B)], dtype=torch.int32, device="cuda")
    ws = torch.empty((ops.topk_workspace_size(B, T, S, k) // 4,), dtype=torch.int32, device="cuda")
    for call in range(2):
        sc = _case(100 * call + B, B, T, S)
        ref = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((B, T, k), -9, dtype=torch.int32, device="cuda")
        ops.topk_select(sc, ref, S, m, pos0, workspace=ws)
        ops.topk_select_noalloc(sc, got, S, m, pos0)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_without_scratch_need_equals_topk_select(ops):
    """A shape that needs no scratch (many short rows) takes the one-CTA path."""
    B, T, S, k, m = 2, 300, 2000, 64, 4
    assert ops.topk_workspace_size(B, T, S, k) == 0
    sc = _case(5, B, T, S)
    pos0 = torch.zeros((B,), dtype=torch.int32, device="cuda")
    ref = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    got = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    ops.topk_select(sc, ref, S, m, pos0)
    ops.topk_select_noalloc(sc, got, S, m, pos0)
    np.testing.assert_array_equal(got.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_shapes_beyond_scratch(ops):
    """512 rows of 1,048,576 entries need ~4.8 MB of histograms: refused."""
    B, T, S, k = 512, 1, 1 << 20, 1024
    assert ops.topk_workspace_size(B, T, S, k) > 1 << 20
    sc = torch.zeros((1,), dtype=torch.bfloat16, device="cuda").as_strided((B, T, S), (0, 0, 0))
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    pos0 = torch.zeros((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(ops.CsaError) as e:
        ops._check("topk_select_noalloc", ops.lib.topk_select_noalloc(
            sc.data_ptr(), ops.CSA_BF16, B, T, S, S, k, 4, 0, pos0.data_ptr(), idx.data_ptr(),
            torch.cuda.current_stream().cuda_stream))
    assert "UNSUPPORTED" in str(e.value)
