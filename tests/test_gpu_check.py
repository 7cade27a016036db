"""Check mode of the layer drivers: csa_validate_indices finds every kind of
bad idx row (an entry outside the visible range, valid entries out of order,
a valid entry after the -1 padding) and reports it in a status word without
trapping; a correct layer run in check mode passes."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_compress_b200 import configs, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import layer
    return layer


def _status(ops, idx, S, m, pos0):
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    ops.validate_indices(idx.cuda(), S, m, pos0.cuda(), st)
    torch.cuda.synchronize()
    return int(st.item())


def test_validate_reports_each_violation(L):
    from long_context_compressed_compress_b200 import ops
    B, T, m, k = 2, 96, 4, 8
    S = T // m
    pos0 = torch.tensor([0, 5], dtype=torch.int32)
    pos = np.arange(T)[None] + pos0.numpy()[:, None]
    sc = np.random.default_rng(3).standard_normal((B, T, S))
    idx = torch.from_numpy(oracle.topk_select(sc, pos, m, k))
    assert _status(ops, idx, S, m, pos0) == 0
    r = 80                                   # sees min(S, 81 // 4) = 20 > k entries
    bad = idx.clone()
    bad[0, r, 3] = 20                        # not visible
    assert _status(ops, bad, S, m, pos0) == 1 | (1 << 8)
    bad = idx.clone()
    bad[1, r, 2], bad[1, r, 3] = idx[1, r, 3], idx[1, r, 2]
    assert _status(ops, bad, S, m, pos0) == 1 | (2 << 8)
    bad = idx.clone()
    bad[0, r, 2] = -1                        # padding, then valid entries
    assert _status(ops, bad, S, m, pos0) == 1 | (3 << 8)
    bad = idx.clone()
    bad[0, 2, 0] = 0                         # row 2 sees no entry: 0 is out of range
    assert _status(ops, bad, S, m, pos0) == 1 | (1 << 8)


def test_check_mode_layer_run_passes(L):
    cfg = configs.scaled(configs.CSA_PREFILL, T=2048, seed=21)
    x = {k: v.cuda() for k, v in inputs.layer_inputs(cfg, device="cpu").items()}
    for fused in (False, True):
        lay = L.CsaPrefill(cfg, chunk=768, fused=fused, check=True)
        lay.run(x)                           # raises if any idx chunk is malformed
        torch.cuda.synchronize()
        assert int(lay.status.item()) == 0
