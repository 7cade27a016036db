"""The prefill split of one sequence over ranks (row shards, compressor and
window halos, all-gathered entries) on one GPU: the ranks run one after the
other in this process (no collective: the gathered entries are the
concatenation of the ranks' compressions), and their outputs together equal
the single-rank layer bit for bit."""
import pytest
import torch

from long_context_compressed_compress_b200 import configs, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods(cuda_ok):
    from long_context_compressed_compress_b200 import build
    build.build()
    from long_context_compressed_compress_b200 import layer, shard
    return layer, shard


@pytest.mark.parametrize("world,T,H", [(2, 4096, 64), (3, 3002, 128), (4, 2048, 64)])
def test_prefill_split_equals_single_rank(mods, world, T, H):
    layer, shard = mods
    cfg = configs.scaled(configs.CSA_PREFILL, T=T, H=H, k=256, seed=41)
    xd = {k: v.cuda() for k, v in inputs.layer_inputs(cfg, device="cpu").items()}
    full = layer.CsaPrefill(cfg).run(xd).clone()
    plan = shard.ShardPlan(cfg.T, cfg.m, cfg.W, world)
    parts = [shard.shard_inputs(xd, plan, r) for r in range(world)]
    lays = [shard.CsaPrefillShard(cfg, plan, r) for r in range(world)]
    ents = [lays[r].compress(parts[r][0], parts[r][1]) for r in range(world)]
    kv_c, k_fp4, k_sf = (torch.cat([e[i] for e in ents], dim=1) for i in range(3))
    outs = [lays[r].attend(parts[r][0], parts[r][2], kv_c, k_fp4, k_sf) for r in range(world)]
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=1)
    assert got.shape == full.shape
    assert torch.equal(got, full)
