"""topk_select_noalloc serves callers that cannot allocate device memory (a
serving loop that must never wait on an allocator, a host runtime that gives
the library no memory of its own): it uses a fixed scratch array inside the
library instead of a caller workspace.  Checked against topk_select with a
workspace and against the oracle's top-k, on two calls in a row.  Kept in its
own file, collected last, and independent of the other tests' state."""
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
        g = got.cpu().numpy()
        np.testing.assert_array_equal(g, ref.cpu().numpy())
        # and against the oracle's selection on the same stored scores (first
        # and last row; the oracle sorts whole rows, so two rows suffice)
        scd = sc.float().cpu().numpy().astype(np.float64)
        pos = pos0.cpu().numpy().astype(np.int64)[:, None] + np.arange(T)[None]
        for (b, t) in ((0, 0), (B - 1, T - 1)):
            want = oracle.topk_select(scd[b:b + 1, t:t + 1], pos[b:b + 1, t:t + 1], m, k)[0, 0]
            np.testing.assert_array_equal(g[b, t], want)


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
    """512 rows of 16,384 entries need about 4.4 MB of histograms, more than the
    1 MiB scratch: the call is refused before any work is queued, and the
    output is left untouched.  The score buffer is real (16 MB), so nothing
    would read out of bounds even if the refusal were missing."""
    B, T, S, k = 512, 1, 16384, 1024
    assert ops.topk_workspace_size(B, T, S, k) > 1 << 20
    sc = torch.zeros((B, T, S), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((B, T, k), -5, dtype=torch.int32, device="cuda")
    pos0 = torch.full((B,), 4 * S, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.CsaError) as e:
        ops.topk_select_noalloc(sc, idx, S, 4, pos0)
    assert "UNSUPPORTED" in str(e.value)
    torch.cuda.synchronize()
    assert bool((idx == -5).all())
