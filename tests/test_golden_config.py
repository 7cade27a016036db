"""The workload definitions use the values the pages print for the layer
(tests/golden/page_config_values.txt, each line with its page and section)."""
import os

from long_context_compressed_compress_b200 import configs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_config_values.txt")


def _values():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kv, cite = line.split("|", 1)
        key, val = (s.strip() for s in kv.split("=", 1))
        assert cite.strip(), key
        out[key] = val
    return out


def test_golden_file_cites_every_value():
    v = _values()
    assert len(v) >= 10


def test_workloads_use_the_printed_values():
    v = _values()
    csa_layers = [configs.CSA_PREFILL] + [c for c in configs.STACK.layers if c.kind == "csa"]
    hca_layers = [configs.HCA_PREFILL] + [c for c in configs.STACK.layers if c.kind == "hca"]
    for c in csa_layers:
        assert c.m == int(v["csa_compress_ratio"])
        assert c.DI == int(v["indexer_rank"])
        assert c.W == int(v["sliding_window"])
        assert c.sink == "normal" and v["attention_sink"] == "true"
    for c in hca_layers:
        assert c.m == int(v["hca_compress_ratio"])
        assert c.W == int(v["sliding_window"])
    # the 1M-context decode and the stack's CSA layers select the printed top-k
    assert configs.CSA_DECODE.k == int(v["csa_top_k"]) and configs.CSA_DECODE.m == int(v["csa_compress_ratio"])
    assert all(c.k == int(v["csa_top_k"]) for c in configs.STACK.layers if c.kind == "csa")
    assert ",".join(c.kind.upper() for c in configs.STACK.layers) == v["layer_pattern"]
    # the 128-head layers (stack, decode) and the variants the pages name
    assert configs.CSA_DECODE.H == int(v["query_heads_large_model"])
    assert configs.HCA_PREFILL_M64.m == int(v["hca_compress_ratio_small_model"])
    assert configs.CSA_PREFILL_K32.k == int(v["csa_top_k_variant"])
    assert configs.CSA_PREFILL_K1024.k == int(v["csa_top_k"])
    # bf16 scores in the bf16 workloads (the fp32 workload keeps fp32 scores)
    assert v["index_score_dtype"] == "bf16" and configs.CSA_PREFILL.dtype == "bf16"


def test_bench_algorithmic_work_closed_forms():
    """The bench's per-launch algorithmic work equals closed forms: visible
    (row, entry) pairs sum min(S, (t+1) // m) over rows; attended rows add
    min(k, visible) + min(W, t + 1); attention FLOPs are 4 D H per attended row."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    c = configs.scaled(configs.CSA_PREFILL, T=1000)
    w = bench.algorithmic_work(c)
    vis = [min(c.S, (t + 1) // c.m) for t in range(c.T)]
    rows = sum(min(c.k, v) + min(c.W, t + 1) for t, v in enumerate(vis))
    assert w["indexer_pairs"] == c.B * sum(vis)
    assert w["attn_rows"] == c.B * rows
    assert w["attn_flops"] == c.B * 4.0 * c.H * c.D * rows
    assert w["topk_bytes"] == c.B * (sum(vis) * 2 + c.T * c.k * 4)
    assert w["indexer_topk_bytes"] == c.B * (c.T * c.HI * (c.DI // 2 + c.DI // 16 + 4) +
                                             c.S * (c.DI // 2 + c.DI // 16) + c.T * c.k * 4)
