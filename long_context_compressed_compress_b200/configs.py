"""The five workloads of the CSA/HCA attention layer, with their sizes.

Names follow the method's notation: B batch, T tokens per sequence, H query heads,
D head / KV dim (one shared KV head, MQA), m compression ratio, S = T // m
compressed entries, H_I x D_I indexer heads x dim, k top-k, W raw window, tau
softmax scale.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class LayerCfg:
    kind: str                 # "csa" or "hca"
    B: int
    T: int
    H: int
    D: int
    m: int
    W: int = 128
    k: int = 0                # CSA top-k
    HI: int = 0               # CSA indexer heads
    DI: int = 0               # CSA indexer dim
    dtype: str = "bf16"       # "bf16" or "f32"
    tau: float = 0.0
    q_scale: float = 1.0      # q ~ N(0,1) * q_scale
    z_std: float = 1.0        # gate logits z ~ N(0, z_std^2)
    sink: str = "normal"      # "normal": sigma_h ~ N(0,1); "zero": sigma_h = 0
    seed: int = 0

    @property
    def S(self) -> int:
        return self.T // self.m


@dataclass(frozen=True)
class DecodeCfg:
    B: int                    # sequences
    T0: int                   # cached tokens before the first decode step
    H: int
    D: int
    HI: int
    DI: int
    k: int
    m: int = 4
    W: int = 128
    steps: int = 64
    dtype: str = "bf16"
    seed: int = 3

    @property
    def S0(self) -> int:
        return self.T0 // self.m

    @property
    def tau(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclass(frozen=True)
class StackCfg:
    layers: tuple = field(default_factory=tuple)
    seed: int = 4


def _csa(**kw):
    kw.setdefault("tau", 1.0 / math.sqrt(kw["D"]))
    return LayerCfg(kind="csa", **kw)


def _hca(**kw):
    kw.setdefault("tau", 1.0 / math.sqrt(kw["D"]))
    return LayerCfg(kind="hca", **kw)


# 1. tiny CSA layer in fp32 (the small case the oracle finishes in seconds)
PR1 = _csa(B=1, T=1024, H=8, D=64, m=4, k=64, HI=2, DI=32, dtype="f32", tau=1.0,
           q_scale=1.0 / 8.0, sink="zero", seed=0)
# 2. CSA prefill, bf16, T = 32K
CSA_PREFILL = _csa(B=1, T=32768, H=64, D=128, m=4, k=512, HI=4, DI=64, seed=1)
# 3. HCA prefill, bf16, 2 x 128K
HCA_PREFILL = _hca(B=2, T=131072, H=64, D=128, m=128, z_std=math.sqrt(2.0), seed=2)
# 4. CSA decode at 1M context: 32 sequences, 262,144 entries each
CSA_DECODE = DecodeCfg(B=32, T0=1 << 20, H=128, D=128, HI=4, DI=64, k=1024)
# 5. four-layer stack HCA, HCA, CSA, CSA at T = 256K, H = 128
STACK = StackCfg(layers=(
    _hca(B=1, T=262144, H=128, D=128, m=128, seed=40),
    _hca(B=1, T=262144, H=128, D=128, m=128, seed=41),
    _csa(B=1, T=262144, H=128, D=128, m=4, k=1024, HI=4, DI=64, seed=42),
    _csa(B=1, T=262144, H=128, D=128, m=4, k=1024, HI=4, DI=64, seed=43),
), seed=4)

WORKLOADS = {
    "pr1_csa_f32": PR1,
    "csa_prefill_32k": CSA_PREFILL,
    "hca_prefill_2x128k": HCA_PREFILL,
    "csa_decode_32x1m": CSA_DECODE,
    "stack_hhcc_256k": STACK,
}


def scaled(cfg: LayerCfg, **kw) -> LayerCfg:
    """A copy of a layer config with some sizes replaced (test cases)."""
    d = dict(cfg.__dict__)
    d.update(kw)
    return LayerCfg(**d)


# Variants of the same kernels named on the pages: HCA ratio 64
# (devpress.csdn.net/awstech/6a462b3a… §3.1) and top-k 32 / 512 / 1024
# (devpress.csdn.net/awstech/6a4623aa… attention paragraph; cf-1.com/news/5231315
# §3.1; yfxerp.com/news/211352 §3 top_k_blocks).
HCA_PREFILL_M64 = scaled(HCA_PREFILL, m=64)
CSA_PREFILL_K32 = scaled(CSA_PREFILL, k=32)
CSA_PREFILL_K1024 = scaled(CSA_PREFILL, k=1024)
WORKLOADS.update({
    "hca_prefill_2x128k_ratio64": HCA_PREFILL_M64,
    "csa_prefill_32k_k32": CSA_PREFILL_K32,
    "csa_prefill_32k_k1024": CSA_PREFILL_K1024,
})
