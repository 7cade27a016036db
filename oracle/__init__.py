"""CPU oracle of the CSA/HCA attention layer (float64 numpy).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s ``cpu_baseline`` / ``--impl reference`` legs may import this
package.  The GPU library never imports it and shares no code with it.

Parity status of each function (what pins it, see ``tests/test_oracle_pins.py``):
  csa_compress, hca_compress  one-hot gates, constant gates, permutation and
                              ratio-1 special cases
  nvfp4_quantize              E4M3 vs torch.float8_e4m3fn; E2M1 vs brute-force
                              nearest-even search; grid round trips
  indexer_score               brute-force loops; one-hot weights; visibility
  topk_select                 brute-force sort on tiny rows with ties and zeros
  sparse_attn / dense_attn    torch SDPA (causal and banded) special cases;
                              k >= S reduces CSA to dense; sink closed form
  swa_sink_merge              split path == fused path
"""
from . import formats  # noqa: F401
from .csa_oracle import *  # noqa: F401,F403
