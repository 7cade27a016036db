"""Host logic of the prefill split (shard.py), on CPU: the shard plan over
random shapes, the window ring's slot mapping, and that the oracle's
compression of each shard with its halo equals the whole-sequence
compression (the exchange the ranks perform, without the collectives)."""
import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from long_context_compressed_compress_b200 import shard


@settings(max_examples=200, deadline=None)
@given(T=st.integers(1, 5000), m=st.sampled_from([1, 2, 4, 8, 64, 128]), W=st.sampled_from([1, 16, 128]),
       world=st.integers(1, 9))
def test_plan_covers_the_sequence_in_whole_blocks(T, m, W, world):
    plan = shard.ShardPlan(T, m, W, world)
    assert plan.start[0] == 0 and plan.end[-1] == T
    for r in range(world):
        s, e = plan.rows(r)
        assert s <= e and s % m == 0
        if r + 1 < world:
            assert e == plan.start[r + 1] and e % m == 0
        # entries of the rank's blocks: consecutive across ranks, all T // m of them
        e0, e1 = plan.entries(r)
        assert e0 == s // m and e1 == e // m
        h0, h1 = plan.raw_halo(r)
        assert h1 == s and h0 == max(0, s - (W - 1))
    assert sum(plan.entries(r)[1] - plan.entries(r)[0] for r in range(world)) == T // m
    # blocks split as evenly as possible: shard sizes (in blocks) differ by at most one
    sizes = [(plan.end[r] - plan.start[r]) // m for r in range(world - 1)] + [plan.entries(world - 1)[1] -
                                                                            plan.entries(world - 1)[0]]
    assert max(sizes) - min(sizes) <= 1


@settings(max_examples=100, deadline=None)
@given(start=st.integers(0, 3000), halo=st.integers(0, 127), rows=st.integers(1, 300),
       W=st.sampled_from([16, 128]))
def test_window_ring_places_token_j_at_slot_j_mod_cap(start, halo, rows, W):
    halo = min(halo, start)
    D = 4
    lo = start - halo
    seq = torch.arange(lo, start + rows, dtype=torch.float32)[None, :, None].repeat(1, 1, D)
    ring = shard.window_ring(seq[:, :halo], seq[:, halo:], start, W)
    cap = ring.shape[1]
    assert cap >= W and cap >= halo + rows
    for j in range(lo, start + rows):
        assert torch.all(ring[0, j % cap] == j)


@pytest.mark.parametrize("T,world", [(1024, 2), (1030, 3), (777, 4)])
def test_shard_compressions_with_halo_equal_the_whole_sequence(T, world):
    m, D = 4, 16
    rng = np.random.default_rng(T + world)
    a, b, z = (rng.standard_normal((1, T, D)) for _ in range(3))
    plan = shard.ShardPlan(T, m, 128, world)
    parts = []
    for r in range(world):
        s, e = plan.rows(r)
        fhp = r > 0
        lo = s - m if fhp else s
        if e - lo < m * (1 + fhp):   # a shard without a complete block emits nothing
            continue
        parts.append(oracle.csa_compress(a[:, lo:e], b[:, lo:e], z[:, lo:e], m, first_has_pred=fhp))
    whole = oracle.csa_compress(a, b, z, m)
    np.testing.assert_array_equal(np.concatenate(parts, axis=1), whole)
