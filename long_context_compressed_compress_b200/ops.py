"""ctypes binding of libcsa_b200.so (declared in include/csa.h).

Argument marshalling only: every function takes torch tensors that already live
on the GPU, passes their data pointers and the current CUDA stream, and raises
``CsaError`` on a non-zero status.  There is no CPU fallback: if the library
is missing the import of this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa_b200.so")

CSA_F32, CSA_BF16 = 0, 1
STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_ALIGNMENT",
          4: "CSA_ERR_CUDA", 5: "CSA_ERR_TIMEOUT"}


class CsaError(RuntimeError):
    def __init__(self, fn, status, cuda_err=0):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}"
                         + (f" (cudaError {cuda_err})" if status == 4 else ""))
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run long_context_compressed_compress_b200.build")
lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
I64 = ctypes.c_int64
SZ = ctypes.c_size_t

_SIGS = {
    "csa_status_string": ([I], ctypes.c_char_p),
    "csa_last_cuda_error": ([], I),
    "csa_version": ([], I),
    "csa_device_status": ([ctypes.POINTER(I)], I),
    "csa_set_wait_timeout_ns": ([ctypes.c_uint64], I),
    "csa_compress": ([P, P, P, I, I, I, I, I, I, P, I, P, I, P, P, F, P], I),
    "hca_compress": ([P, P, I, I, I, I, I, P, I, P], I),
    "nvfp4_quantize": ([P, I, I64, I, F, P, P, P], I),
    "indexer_score": ([P, P, F, P, P, F, P, I, I, I, I, I, I, I, I, I, P, P, I, I, P, P], I),
    "topk_select": ([P, I, I, I, I, I, I, I, I, P, P, P, SZ, P], I),
    "indexer_topk": ([P, P, F, P, P, F, P, I, I, I, I, I, I, I, I, I, P, P, I, P, P], I),
    "indexer_topk_max_entries": ([I, I], I),
    "csa_validate_indices": ([P, I, I, I, I, I, I, P, P, P], I),
    "topk_workspace_size": ([I, I, I, I], SZ),
    "topk_select_noalloc": ([P, I, I, I, I, I, I, I, I, P, P, P], I),
    "sparse_attn_fwd": ([P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, P, P, P, I, P, P], I),
    "hca_dense_attn_fwd": ([P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, I, P, P, P, I, P, P], I),
    "swa_sink_merge": ([P, P, P, P, P, F, I, I, I, I, I, I, I, I, P, P, I, P], I),
    "csa_ring_append": ([P, I, I, I, P, I, P, P], I),
    "csa_pos_advance": ([P, I, I, P], I),
    "csa_decode_update": ([P] * 8 + [I] * 8 + [P] * 12 + [F, P, P], I),
    "csa_state_gather": ([P, I, I, I, I, P, I, I, I, P, I, P], I),
    "grouped_out_proj": ([P, I, I, I, I, I, P, P, I, P, P, P, P], I),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTS = tuple(_SIGS)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _dt(t_or_dtype):
    d = t_or_dtype.dtype if isinstance(t_or_dtype, torch.Tensor) else t_or_dtype
    if d == torch.float32:
        return CSA_F32
    if d == torch.bfloat16:
        return CSA_BF16
    raise ValueError(f"unsupported dtype {d}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(fn, st):
    if st != 0:
        raise CsaError(fn, st, lib.csa_last_cuda_error())


def device_status():
    """Read and clear the library's per-device status word (calls given no
    status word of their own report a timed-out wait there)."""
    v = I(0)
    _check("csa_device_status", lib.csa_device_status(ctypes.byref(v)))
    return v.value


def set_wait_timeout_ns(ns):
    """Wall-time limit of the kernels' bounded waits (0 = the default 2 s)."""
    _check("csa_set_wait_timeout_ns", lib.csa_set_wait_timeout_ns(int(ns)))


def csa_compress(a, b, z, m, out=None, out_fp4=None, out_sf=None, gscale=1.0, first_has_pred=0,
                 ring_pos=None, out_bstride=0, out_dtype=None, stream=None):
    B, T, D = a.shape[-3], a.shape[-2], a.shape[-1]
    od = _dt(out) if out is not None else _dt(out_dtype if out_dtype is not None else a.dtype)
    _check("csa_compress", lib.csa_compress(
        _ptr(a), _ptr(b), _ptr(z), _dt(a), B, T, D, m, first_has_pred, _ptr(ring_pos), out_bstride,
        _ptr(out), od, _ptr(out_fp4), _ptr(out_sf), gscale, _stream(stream)))


def hca_compress(a, z, m, out, stream=None):
    B, T, D = a.shape
    _check("hca_compress", lib.hca_compress(_ptr(a), _ptr(z), _dt(a), B, T, D, m, _ptr(out), _dt(out),
                                            _stream(stream)))


def nvfp4_quantize(x, packed, sf, gscale=1.0, stream=None):
    D = x.shape[-1]
    rows = x.numel() // D
    _check("nvfp4_quantize", lib.nvfp4_quantize(_ptr(x), _dt(x), rows, D, gscale, _ptr(packed), _ptr(sf),
                                                _stream(stream)))


def indexer_score(q_fp4, q_sf, k_fp4, k_sf, w, q_pos0, score, S, m, row0=0, T_chunk=None, q_gscale=1.0,
                  k_gscale=1.0, status=None, stream=None):
    """q_fp4 [B,T,HI,DI/2], k_fp4 [B,k_bstride,DI/2], w [B,T,HI], score [B,T_chunk,ld]."""
    B, T, HI, half = q_fp4.shape
    DI = half * 2
    T_chunk = T - row0 if T_chunk is None else T_chunk
    _check("indexer_score", lib.indexer_score(
        _ptr(q_fp4), _ptr(q_sf), q_gscale, _ptr(k_fp4), _ptr(k_sf), k_gscale, _ptr(w), B, T, row0, T_chunk,
        S, k_fp4.shape[1], HI, DI, m, _ptr(q_pos0), _ptr(score), _dt(score), score.shape[-1],
        _ptr(status), _stream(stream)))


def topk_select(score, idx, S, m, q_pos0, row0=0, workspace=None, stream=None):
    B, T_chunk, ld = score.shape
    k = idx.shape[-1]
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("topk_select", lib.topk_select(_ptr(score), _dt(score), B, T_chunk, S, ld, k, m, row0,
                                          _ptr(q_pos0), _ptr(idx), _ptr(workspace), ws, _stream(stream)))


def indexer_topk(q_fp4, q_sf, k_fp4, k_sf, w, q_pos0, idx, S, m, row0=0, T_chunk=None, q_gscale=1.0,
                 k_gscale=1.0, status=None, stream=None):
    """Indexer score and top-k in one kernel: idx [B,T_chunk,k] equals
    topk_select of the BF16 scores indexer_score would write."""
    B, T, HI, half = q_fp4.shape
    DI = half * 2
    T_chunk = T - row0 if T_chunk is None else T_chunk
    _check("indexer_topk", lib.indexer_topk(
        _ptr(q_fp4), _ptr(q_sf), q_gscale, _ptr(k_fp4), _ptr(k_sf), k_gscale, _ptr(w), B, T, row0, T_chunk,
        S, k_fp4.shape[1], HI, DI, m, _ptr(q_pos0), _ptr(idx), idx.shape[-1], _ptr(status), _stream(stream)))


def indexer_topk_max_entries(HI, DI):
    return int(lib.indexer_topk_max_entries(HI, DI))


def validate_indices(idx, S, m, q_pos0, status, row0=0, stream=None):
    """Check idx [B, T_chunk, k] (entries in [0, visible), ascending, then -1);
    a violation is recorded in the device word ``status`` (int32 [1])."""
    B, T_chunk, k = idx.shape
    _check("csa_validate_indices", lib.csa_validate_indices(_ptr(idx), B, T_chunk, k, S, m, row0, _ptr(q_pos0),
                                                            _ptr(status), _stream(stream)))


def topk_select_noalloc(score, idx, S, m, q_pos0, row0=0, stream=None):
    """topk_select without a workspace: the library's fixed scratch serves the
    multi-CTA path (see the C header for its size limit and concurrency rule)."""
    B, T_chunk, ld = score.shape
    k = idx.shape[-1]
    _check("topk_select_noalloc", lib.topk_select_noalloc(_ptr(score), _dt(score), B, T_chunk, S, ld, k, m, row0,
                                                          _ptr(q_pos0), _ptr(idx), _stream(stream)))


def topk_workspace_size(B, T_chunk, S, k):
    return int(lib.topk_workspace_size(B, T_chunk, S, k))


def sparse_attn_fwd(q, kv_c, idx, kv_raw, sink, tau, W, q_pos0, out, lse=None, row0=0, T_chunk=None,
                    raw_cap=None, status=None, stream=None):
    B, T, H, D = q.shape
    T_chunk = T - row0 if T_chunk is None else T_chunk
    raw_cap = (kv_raw.shape[1] if kv_raw is not None else 1) if raw_cap is None else raw_cap
    _check("sparse_attn_fwd", lib.sparse_attn_fwd(
        _ptr(q), _ptr(kv_c), _ptr(idx), _ptr(kv_raw), _ptr(sink), tau, W, B, T, row0, T_chunk, H, D,
        kv_c.shape[1], idx.shape[-1], raw_cap, _ptr(q_pos0), _ptr(out), _ptr(lse), _dt(q), _ptr(status),
        _stream(stream)))


def hca_dense_attn_fwd(q, kv_c, kv_raw, sink, tau, W, q_pos0, out, m, S=None, lse=None, row0=0, T_chunk=None,
                       raw_cap=None, status=None, stream=None):
    B, T, H, D = q.shape
    T_chunk = T - row0 if T_chunk is None else T_chunk
    S = kv_c.shape[1] if S is None else S
    raw_cap = (kv_raw.shape[1] if kv_raw is not None else 1) if raw_cap is None else raw_cap
    _check("hca_dense_attn_fwd", lib.hca_dense_attn_fwd(
        _ptr(q), _ptr(kv_c), _ptr(kv_raw), _ptr(sink), tau, W, B, T, row0, T_chunk, H, D, kv_c.shape[1], S, m,
        raw_cap, _ptr(q_pos0), _ptr(out), _ptr(lse), _dt(q), _ptr(status), _stream(stream)))


def swa_sink_merge(o_c, lse_c, q, kv_raw, sink, tau, W, q_pos0, out, row0=0, T_chunk=None, raw_cap=None,
                   stream=None):
    B, T, H, D = q.shape
    T_chunk = T - row0 if T_chunk is None else T_chunk
    raw_cap = kv_raw.shape[1] if raw_cap is None else raw_cap
    _check("swa_sink_merge", lib.swa_sink_merge(
        _ptr(o_c), _ptr(lse_c), _ptr(q), _ptr(kv_raw), _ptr(sink), tau, W, B, T, row0, T_chunk, H, D, raw_cap,
        _ptr(q_pos0), _ptr(out), _dt(q), _stream(stream)))


def csa_ring_append(rows, ring, pos, stream=None):
    B, D = rows.shape
    _check("csa_ring_append", lib.csa_ring_append(_ptr(rows), _dt(rows), B, D, _ptr(ring), ring.shape[1],
                                                  _ptr(pos), _stream(stream)))


def csa_decode_update(x, carry, ring, kv_c, k_fp4, k_sf, q_fp4, q_sf, pos, m, gscale=1.0, stream=None):
    """One decode step's cache update in one launch (see the C header):
    ``x`` holds this step's rows a, b, z, a_I, b_I, z_I, kv_raw [B, .] and
    q_I [B, HI, DI]; ``carry`` the six 2m-slot carry rings by name."""
    B, D = x["a"].shape[0], x["a"].shape[-1]
    DI = x["a_I"].shape[-1]
    HI = x["q_I"].shape[-2]
    names = ("a", "b", "z", "a_I", "b_I", "z_I")
    _check("csa_decode_update", lib.csa_decode_update(
        *[_ptr(x[n]) for n in names], _ptr(x["kv_raw"]), _ptr(x["q_I"]), _dt(x["a"]), B, D, DI, HI, m,
        ring.shape[1], kv_c.shape[1], *[_ptr(carry[n]) for n in names], _ptr(ring), _ptr(kv_c), _ptr(k_fp4),
        _ptr(k_sf), _ptr(q_fp4), _ptr(q_sf), gscale, _ptr(pos), _stream(stream)))


def csa_pos_advance(pos, delta=1, stream=None):
    _check("csa_pos_advance", lib.csa_pos_advance(_ptr(pos), pos.numel(), delta, _stream(stream)))


def csa_state_gather(src, pos, dst, m=0, nrows=0, src_cap=None, stream=None):
    """Snapshot rows of a ring or a [B, T, D] stream into dst [B, npos, cap, D]
    (see include/csa.h): window mode (m = 0, the last ``nrows`` tokens up to
    pos) or carry mode (m >= 1, the last complete block and the one in
    progress).  pos: int32 [B, npos] on the device."""
    B, cap_src, D = src.shape
    npos = pos.shape[-1]
    dst_cap = dst.shape[-2]
    _check("csa_state_gather", lib.csa_state_gather(
        _ptr(src), _dt(src), B, D, cap_src if src_cap is None else src_cap, _ptr(pos), npos, m, nrows,
        _ptr(dst), dst_cap, _stream(stream)))


def grouped_out_proj(o, w1, w2, y, out, status=None, stream=None):
    """o [..., H, D] bf16 -> y [M, g*d_g], out [M, d_model] (see include/csa.h);
    w1 [g, d_g, (H/g)*D], w2 [d_model, g*d_g]."""
    H, D = o.shape[-2], o.shape[-1]
    M = o.numel() // (H * D)
    g, d_g, _ = w1.shape
    _check("grouped_out_proj", lib.grouped_out_proj(
        _ptr(o), M, H, D, g, d_g, _ptr(w1), _ptr(w2), w2.shape[0], _ptr(y), _ptr(out), _ptr(status),
        _stream(stream)))
