"""Host-side checks of the C ABI (no GPU needed): the library builds, loads, and
exports every function that include/csa.h declares; argument validation
rejects bad calls before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from long_context_compressed_compress_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "csa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+([a-z_0-9]+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_hot_path_entry_points():
    names = _declared_functions()
    for fn in ("csa_compress", "hca_compress", "nvfp4_quantize", "indexer_score", "topk_select",
               "sparse_attn_fwd", "hca_dense_attn_fwd", "swa_sink_merge"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"missing export {name}"


def test_binding_covers_every_declared_symbol(lib):
    from long_context_compressed_compress_b200 import ops
    assert set(_declared_functions()) <= set(ops.EXPORTS)


def test_status_strings_and_version(lib):
    lib.csa_status_string.restype = ctypes.c_char_p
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert lib.csa_status_string(5) == b"CSA_ERR_TIMEOUT"
    assert lib.csa_version() >= 100


def test_argument_validation_rejects_before_launch(lib):
    """Null pointers, unsupported dims and misalignment return an error code
    without touching the device (no GPU in this process)."""
    from long_context_compressed_compress_b200 import ops
    L = ops.lib
    # null inputs
    assert L.csa_compress(None, None, None, 1, 1, 8, 128, 4, 0, None, 0, None, 1, None, None, 1.0, None) == 1
    assert L.hca_compress(None, None, 1, 1, 128, 128, 128, None, 1, None) == 1
    fake = 1 << 20                      # aligned fake address; never dereferenced
    # D not a multiple of 16 for NVFP4
    assert L.nvfp4_quantize(fake, 1, 4, 24, 1.0, fake, fake, None) == 2
    # misaligned input
    assert L.nvfp4_quantize(fake + 2, 1, 4, 32, 1.0, fake, fake, None) == 3
    # non-positive global scale
    assert L.nvfp4_quantize(fake, 1, 4, 32, 0.0, fake, fake, None) == 1
    # indexer: unsupported DI / HI
    assert L.indexer_score(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 4, 48, 4, fake, fake,
                           1, 16, None, None) == 2
    assert L.indexer_score(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 3, 64, 4, fake, fake,
                           1, 16, None, None) == 2
    # fused indexer + top-k: DI other than 64, HI outside {4, 8}, null idx, k < 1
    assert L.indexer_topk(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 4, 32, 4, fake, fake, 8,
                          None, None) == 2
    assert L.indexer_topk(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 2, 64, 4, fake, fake, 8,
                          None, None) == 2
    assert L.indexer_topk(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 4, 64, 4, fake, None, 8,
                          None, None) == 1
    assert L.indexer_topk(fake, fake, 1.0, fake, fake, 1.0, fake, 1, 64, 0, 64, 16, 16, 4, 64, 4, fake, fake, 0,
                          None, None) == 1
    assert L.indexer_topk_max_entries(4, 32) == 0
    # fused decode update: fp32 rows take the separate calls
    assert L.csa_decode_update(*([fake] * 8), 0, 1, 128, 64, 4, 4, 128, 64, *([fake] * 12), 1.0, fake, None) == 2
    # attention: unsupported head dim
    assert L.sparse_attn_fwd(fake, fake, fake, fake, None, 1.0, 128, 1, 256, 0, 256, 8, 96, 64, 8, 256, fake,
                             fake, None, 1, None, None) == 2
    # window larger than the ring
    assert L.hca_dense_attn_fwd(fake, fake, fake, None, 1.0, 128, 1, 256, 0, 256, 8, 64, 2, 2, 128, 64, fake,
                                fake, None, 1, None, None) == 1
    # top-k: ld < S
    assert L.topk_select(fake, 1, 1, 4, 64, 32, 8, 4, 0, fake, fake, None, 0, None) == 1
    # empty problems are a no-op success
    assert L.topk_select(fake, 1, 0, 4, 64, 64, 8, 4, 0, fake, fake, None, 0, None) == 0
    # the wait limit is a host setting (no device access)
    assert L.csa_set_wait_timeout_ns(0) == 0


def test_binding_argument_counts_match_the_header():
    """Every binding's argtypes list has as many entries as the C declaration
    has parameters (a short list would shift every argument after it)."""
    from long_context_compressed_compress_b200 import ops
    txt = open(os.path.join(ROOT, "include", "csa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    decls = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+([a-z_0-9]+)\s*\(([^;]*?)\)\s*;", txt,
                       flags=re.M | re.S)
    assert len(decls) >= 15
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        assert len(ops._SIGS[name][0]) == n, (name, n, len(ops._SIGS[name][0]))
