"""KV-cache state management (cf-1.com/news/5231315 §4.4: sliding-window
checkpoints every 1024 tokens and restoring a shared prefix): snapshots taken
from a prefill's inputs are compared bit for bit with the rows they must
hold, and a decode restored from a snapshot (the prefill's compressed entries
and NVFP4 keys as its cache) is compared with the oracle's decode started from
the oracle's own prefill state, step by step."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_compress_b200 import configs, inputs
from test_gpu_decode import check_step

pytestmark = pytest.mark.gpu

CARRY = ("a", "b", "z", "a_I", "b_I", "z_I")


@pytest.fixture(scope="module")
def L(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import layer
    return layer


def _np(t):
    return t.detach().cpu().to(torch.float64).numpy()


def oracle_state(x, T0, m, W):
    """The oracle's decode state after a prefill of tokens [0, T0): entries of
    completed blocks, their NVFP4 keys, the raw window and the carry."""
    f = {k: v.to(torch.float64).numpy() for k, v in x.items()}
    B = f["a"].shape[0]
    st = {"kv_c": oracle.round_out(oracle.csa_compress(f["a"][:, :T0], f["b"][:, :T0], f["z"][:, :T0], m), "bf16")}
    ks = oracle.round_out(oracle.csa_compress(f["a_I"][:, :T0], f["b_I"][:, :T0], f["z_I"][:, :T0], m), "bf16")
    st["khat"] = oracle.nvfp4_quantize(ks)["xhat"]
    st["ring"] = np.zeros((B, W, f["kv_raw"].shape[-1]))
    for j in range(max(0, T0 - W), T0):
        st["ring"][:, j % W] = f["kv_raw"][:, j]
    for n in CARRY:
        c = np.zeros((B, 2 * m, f[n].shape[-1]))
        for j in range(max(0, (T0 // m - 1) * m), T0):
            c[:, j % (2 * m)] = f[n][:, j]
        st["carry_" + n] = c
    return st


def test_snapshot_contents_bit_exact(L):
    """Window and carry snapshots at p = 1023, 2047, 3071 of two sequences
    hold exactly the rows the decode layout puts there (zeros elsewhere)."""
    cfg = configs.scaled(configs.CSA_PREFILL, B=2, T=3 * 1024 + 100, seed=31)
    x = inputs.layer_inputs(cfg, device="cpu")
    xd = {k: v.cuda() for k, v in x.items()}
    ck = L.PrefixCheckpoints(cfg, xd, every=1024)
    torch.cuda.synchronize()
    assert ck.positions == [1023, 2047, 3071]
    m, W = cfg.m, cfg.W
    for i, p in enumerate(ck.positions):
        want = np.zeros((cfg.B, W, cfg.D))
        for j in range(p - W + 1, p + 1):
            want[:, j % W] = _np(x["kv_raw"][:, j])
        np.testing.assert_array_equal(_np(ck.ring[:, i]), want)
        lo = m * ((p + 1) // m - 1)
        for n in CARRY:
            want = np.zeros((cfg.B, 2 * m, x[n].shape[-1]))
            for j in range(lo, p + 1):
                want[:, j % (2 * m)] = _np(x[n][:, j])
            np.testing.assert_array_equal(_np(ck.carry[n][:, i]), want)


@pytest.mark.parametrize("snap,H", [(1, 64), (0, 128)])
def test_prefill_checkpoint_restore_decode(L, snap, H):
    """Prefill T tokens on the GPU, take the every-1024 snapshots, restore the
    decode state at snapshot ``snap`` (next token 1024 (snap + 1)) and decode
    nine tokens; each step equals the oracle's decode step from the oracle's
    prefill state (index sets up to near-ties, outputs within 2e-2).  The
    steps cross a block boundary, so entries are emitted into the restored
    cache."""
    cfg = configs.scaled(configs.CSA_PREFILL, B=2, H=H, k=128, T=2 * 1024 + 40, seed=32)
    x = inputs.layer_inputs(cfg, device="cpu")
    xd = {k: v.cuda() for k, v in x.items()}
    pre = L.CsaPrefill(cfg)
    pre.run(xd)
    ck = L.PrefixCheckpoints(cfg, xd, every=1024)
    p = ck.positions[snap]
    T0 = p + 1
    dcfg = dataclasses.replace(configs.CSA_DECODE, B=cfg.B, T0=T0, H=cfg.H, k=cfg.k, steps=9, seed=33)
    dec = ck.restore(dcfg, snap, pre.kv_c, pre.k_fp4, pre.k_sf, extra_entries=4, with_lse=True)
    st_o = oracle_state(x, T0, cfg.m, cfg.W)
    sink = x["sink"]
    seqs = list(range(cfg.B))
    for step in range(9):
        xs = inputs.decode_step_inputs(dcfg, step)
        xs["sink"] = sink
        dec.step({k: v.cuda() for k, v in xs.items()})
        torch.cuda.synchronize()
        xo = {k: _np(v) for k, v in xs.items()}
        ref = oracle.csa_decode_step(st_o, xo, T0 + step, cfg.m, cfg.k, cfg.W, cfg.tau, cfg.dtype)
        gi = dec.idx.cpu().numpy()[:, 0]
        go = _np(dec.out)[:, 0]
        gl = dec.lse.cpu().numpy()[:, 0].astype(np.float64)
        check_step(gi, go, gl, ref, st_o, xo, T0 + step, dcfg)
