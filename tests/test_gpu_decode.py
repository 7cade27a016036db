"""Decode-step parity: the GPU decode driver (C-ABI calls, eager and replayed
from a CUDA graph) against the oracle's decode step, on the synthetic 1M-context
cache recipe (reduced context here, full size on a sample of sequences below).

Acceptance as for prefill: index sets agree up to near-ties (2 bf16 ulps of the
k-th score), outputs within 2e-2 max-abs with the oracle's attention fed the
GPU's indices, and end to end where the index sets agree.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle import formats
from long_context_compressed_compress_b200 import configs, inputs

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


def oracle_state(st, cfg, seqs):
    """float64 oracle state for the sequences ``seqs`` of a drawn decode cache."""
    S0 = cfg.S0
    o = {"kv_c": _np(st["kv_c"][seqs, :S0]),
         "khat": oracle.nvfp4_quantize(_np(st["k_I_src"][seqs, :S0]))["xhat"],
         "ring": _np(st["ring"][seqs]).copy()}
    slot0 = ((cfg.T0 // cfg.m - 1) % 2) * cfg.m
    for n in CARRY:
        src = _np(st["carry_" + n][seqs])
        buf = np.zeros((len(seqs), 2 * cfg.m, src.shape[-1]))
        buf[:, slot0:slot0 + cfg.m] = src
        o["carry_" + n] = buf
    return o


def check_step(got_idx, got_out, got_lse, ref, st_o, x, p, cfg):
    """Index sets (overlap and near-tie rule), attention on the GPU's indices,
    and end to end on the sequences whose index sets agree."""
    B = got_idx.shape[0]
    agree, overlap = [], []
    for b in range(B):
        ro = set(ref["idx"][b][ref["idx"][b] >= 0].tolist())
        go = set(got_idx[b][got_idx[b] >= 0].tolist())
        agree.append(ro == go)
        overlap.append(1.0 if not ro and not go else len(ro & go) / max(1, len(ro)))
        if ro != go:
            sc = ref["score"][b]
            kth = np.sort(sc[list(ro)])[0]
            tol = 2 * formats.bf16(abs(kth)) * 2.0 ** -8
            for s in ro ^ go:
                assert abs(sc[s] - kth) <= tol, f"seq {b}: entry {s} score {sc[s]} vs k-th {kth}"
    assert np.mean(overlap) >= 0.995
    q = x["q"][:, None]
    pos = np.full((B, 1), p)
    o2, l2 = oracle.sparse_attn(q, st_o["kv_c"], got_idx[:, None], st_o["ring"], cfg.W, x["sink"], cfg.tau,
                                cfg.W, pos)
    o2 = oracle.round_out(o2, cfg.dtype)[:, 0]
    assert np.abs(got_out - o2).max() <= 2e-2
    l2 = formats.f32(l2)[:, 0]
    assert np.abs(got_lse - l2).max() <= 2.0 ** -8 * max(1.0, np.abs(l2).max())
    for b in range(B):
        if agree[b]:
            assert np.abs(got_out[b] - ref["out"][b]).max() <= 2e-2


def run_decode(L, cfg, seqs, n_steps, graph):
    """Run ``n_steps`` decode steps for every sequence on the GPU and check the
    sequences ``seqs`` against the oracle after each step."""
    st = inputs.decode_state(cfg)
    st_o = oracle_state(st, cfg, seqs)
    sink = _np(st["sink"])
    if graph:
        x0 = {k: v.cuda() for k, v in inputs.decode_step_inputs(cfg, 0).items()}
        warm = L.CsaDecode(cfg, {k: v.cuda() for k, v in st.items()}, cfg.T0)
        warm.step(x0)                  # first-call set-up happens outside the capture
        torch.cuda.synchronize()
        del warm
        lay = L.CsaDecode(cfg, {k: v.cuda() for k, v in st.items()}, cfg.T0, with_lse=True)
        lay.capture(x0)
    else:
        lay = L.CsaDecode(cfg, {k: v.cuda() for k, v in st.items()}, cfg.T0, with_lse=True)
    results = []
    for step in range(n_steps):
        p = cfg.T0 + step
        x = inputs.decode_step_inputs(cfg, step)
        if graph:
            for k, v in x.items():
                lay.x[k].copy_(v)
            lay.replay()
        else:
            lay.step({k: v.cuda() for k, v in x.items()})
        torch.cuda.synchronize()
        xo = {k: _np(v[seqs]) for k, v in x.items()}
        xo["sink"] = sink
        ref = oracle.csa_decode_step(st_o, xo, p, cfg.m, cfg.k, cfg.W, cfg.tau, cfg.dtype)
        gi = lay.idx.cpu().numpy()[seqs, 0]
        go = _np(lay.out)[seqs, 0]
        gl = lay.lse.cpu().numpy()[seqs, 0].astype(np.float64)
        check_step(gi, go, gl, ref, st_o, xo, p, cfg)
        results.append((gi, go))
    return results


SMALL = dataclasses.replace(configs.CSA_DECODE, B=3, T0=1 << 16, steps=8)


def test_decode_steps_match_oracle(L):
    """Six steps from T0 = 65536 (entries 16384.., multi-CTA top-k rows, k=1024):
    step 3 completes a block, so an entry is emitted and becomes visible."""
    run_decode(L, SMALL, [0, 1, 2], 6, graph=False)


def test_decode_graph_replay_equals_eager(L):
    eager = run_decode(L, SMALL, [0, 1, 2], 5, graph=False)
    replay = run_decode(L, SMALL, [0, 1, 2], 5, graph=True)
    for (i1, o1), (i2, o2) in zip(eager, replay):
        np.testing.assert_array_equal(i1, i2)
        np.testing.assert_array_equal(o1, o2)


def test_decode_full_size_sampled(L):
    """32 sequences x 1,048,576 cached tokens (262,144 entries), H=128, k=1024:
    the GPU runs all sequences; the oracle checks sequences 0, 13 and 31 over
    four steps (the fourth emits an entry)."""
    run_decode(L, configs.CSA_DECODE, [0, 13, 31], 4, graph=False)


def test_decode_from_empty_cache(L):
    """Twelve steps from position 0 with an empty cache: the window is partly
    empty, no entry is visible before p = 3, and p = 3 emits entry 0, whose
    softmax covers only its own block's m logits (no predecessor)."""
    cfg = dataclasses.replace(configs.CSA_DECODE, B=3, T0=0, steps=12)
    run_decode(L, cfg, [0, 1, 2], 12, graph=False)


def test_fused_state_update_equals_separate_calls(L):
    """csa_decode_update (one launch) leaves the carry rings, the window ring,
    the compressed entries, their NVFP4 keys and q_I's NVFP4 codes exactly as
    the seven appends, two decode-mode compressions and the quantisation do,
    over eight steps (two entries emitted), from an empty cache and from a
    cache of 65536 tokens; the step outputs are identical."""
    for cfg in (dataclasses.replace(configs.CSA_DECODE, B=3, T0=0, steps=8), SMALL):
        st = inputs.decode_state(cfg)
        lays = [L.CsaDecode(cfg, {k: v.cuda() for k, v in st.items()}, cfg.T0, fused_update=f) for f in (True, False)]
        assert lays[0].fused_update and not lays[1].fused_update
        assert lays[0].launches < lays[1].launches
        for step in range(8):
            x = {k: v.cuda() for k, v in inputs.decode_step_inputs(cfg, step).items()}
            outs = [lay.step(x).clone() for lay in lays]
            torch.cuda.synchronize()
            f, s = lays
            for n in CARRY:
                assert torch.equal(f.carry[n], s.carry[n]), n
            for name in ("ring", "kv_c", "k_fp4", "k_sf", "q_fp4", "q_sf", "idx", "pos"):
                assert torch.equal(getattr(f, name), getattr(s, name)), (step, name)
            assert torch.equal(outs[0], outs[1])
