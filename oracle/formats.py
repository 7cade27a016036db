"""Number formats used by the CSA/HCA path, written from their published definitions.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` use the oracle.

Formats (sign-magnitude, round-to-nearest-even, saturating to the largest finite
value, as the OCP "Microscaling Formats (MX) v1.0" specification and NVIDIA's
NVFP4 description define them):

* FP8 E4M3 ("fn" variant): 4 exponent bits, bias 7, 3 mantissa bits, no infinity,
  largest finite 448, smallest normal 2^-6, subnormal step 2^-9.
* FP4 E2M1: 2 exponent bits, bias 1, 1 mantissa bit, no infinity / NaN,
  representable magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* BF16: 8 exponent bits, bias 127, 7 stored mantissa bits (fp32 range).
* FP32: IEEE binary32.

The lightning indexer quantises its QK path to FP4 with per-16-element block
scales (cf-1.com/news/5231315, §3.4 "两个降开销的设计" and §4.4 "FP4 QAT 与 KV Cache
层级"; the 16-element block and E4M3 scales are the NVFP4 format named for the
indexer keys).  The index scores are stored in BF16 (same page, §4.4).

Every rounding below works on float64 inputs that hold the exact value to be
rounded, and rounds exactly once.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_rne_sat", "e4m3", "e2m1", "bf16", "f32",
    "E2M1_VALUES", "e2m1_code", "e4m3_code", "e4m3_decode", "e2m1_decode",
]


def round_rne_sat(v, mant_bits: int, emin: int, maxfinite: float):
    """Round each float64 in ``v`` to the binary format with ``mant_bits`` stored
    mantissa bits, minimum normal exponent ``emin`` (gradual underflow below it),
    nearest-even on ties, clamped to +-maxfinite.  NaN stays NaN.

    The quantum of a value x with 2^E <= |x| < 2^(E+1) is 2^(E - mant_bits), with
    E clamped below at emin (subnormals share the smallest normal binade's quantum).
    Dividing by a power of two and ``np.rint`` (ties to even) are exact in float64
    for every input these formats see, so this is a single correct rounding.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    mag = np.abs(v)
    nz = mag > 0
    # frexp: mag = f * 2^e with 0.5 <= f < 1, so floor(log2(mag)) = e - 1 exactly.
    _, e = np.frexp(mag[nz])
    E = np.maximum(e.astype(np.int64) - 1, emin)
    quantum = np.ldexp(1.0, E - mant_bits)
    r = np.rint(mag[nz] / quantum) * quantum
    out[nz] = np.minimum(r, maxfinite)
    out = np.copysign(out, v)
    out[np.isnan(v)] = np.nan
    return out


def e4m3(v):
    """FP8 E4M3 (fn): RNE, saturate to +-448."""
    return round_rne_sat(v, 3, -6, 448.0)


def e2m1(v):
    """FP4 E2M1: RNE, saturate to +-6."""
    return round_rne_sat(v, 1, 0, 6.0)


def bf16(v):
    """BF16: RNE.  Values beyond the bf16 range do not occur on this path."""
    return round_rne_sat(v, 7, -126, float(np.finfo(np.float32).max))


def f32(v):
    """IEEE binary32 RNE (numpy's float64->float32 cast is correctly rounded)."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


# --- bit codes ---------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _all_e4m3_values():
    vals = np.zeros(256)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        ex = (code >> 3) & 0xF
        mt = code & 0x7
        if ex == 0xF and mt == 0x7:
            vals[code] = np.nan               # the single NaN pattern (per sign)
        elif ex == 0:
            vals[code] = s * mt * 2.0 ** -9    # subnormal: mt/8 * 2^-6
        else:
            vals[code] = s * (1.0 + mt / 8.0) * 2.0 ** (ex - 7)
    return vals


_E4M3_TABLE = _all_e4m3_values()


def e4m3_decode(codes):
    return _E4M3_TABLE[np.asarray(codes, dtype=np.int64)]


def e2m1_decode(codes):
    codes = np.asarray(codes, dtype=np.int64)
    mag = E2M1_VALUES[codes & 0x7]
    return np.where(codes & 0x8, -mag, mag)


def e4m3_code(vals):
    """Bit pattern of values that are already exactly E4M3 (non-NaN).  -0 and +0
    both map to 0x00, the pattern a round-to-nearest conversion of +0 yields."""
    vals = np.asarray(vals, dtype=np.float64)
    mag = np.abs(vals)
    pos = _E4M3_TABLE[:127]                     # codes 0x00..0x7E, increasing
    idx = np.searchsorted(pos, mag)
    idx = np.minimum(idx, 126)
    if not np.all(pos[idx] == mag):
        raise ValueError("value not representable in E4M3")
    sign = (vals < 0) & (mag > 0)
    return (idx | (sign.astype(np.int64) << 7)).astype(np.uint8)


def e2m1_code(vals):
    """4-bit pattern (sign << 3 | exp << 1 | mantissa) of exact E2M1 values.
    -0 maps to the negative-zero pattern 0x8 only if the value is negative zero."""
    vals = np.asarray(vals, dtype=np.float64)
    mag = np.abs(vals)
    idx = np.searchsorted(E2M1_VALUES, mag)
    idx = np.minimum(idx, 7)
    if not np.all(E2M1_VALUES[idx] == mag):
        raise ValueError("value not representable in E2M1")
    sign = np.signbit(vals)
    return (idx | (sign.astype(np.int64) << 3)).astype(np.uint8)
