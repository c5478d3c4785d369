"""FP8 E4M3 codec and per-row absmax quantiser (oracle side; test infrastructure).

The pages only say that the indexer key path is quantised to FP8 before it is
written to the cache ("Study MLA Indexer", section "数学流": ``quant(FP8)`` on the
K compressor output; "Lightning Indexer 详解" §1: the indexer "可 FP8 实现").  They
fix neither the FP8 format nor the scale granularity, so this module takes the
plainest reading:

* format: OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6; there are no
  infinities; S.1111.111 is NaN; the largest finite magnitude is
  S.1111.110 = 1.75 * 2^8 = 448.
* encode: round to nearest, ties to even, then saturate to +-448 (satfinite).
* scale: one fp32 scale per row, ``scale = fp32(absmax) / 448`` (IEEE fp32
  division); the stored code of x is ``encode(fp32(x) / scale)`` (again IEEE fp32
  division).  An all-zero row gets scale 1 and all-zero codes.

The decoded value of a code c with row scale s is ``value(c) * s``, exact in fp64.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0          # 1.75 * 2^8, the largest finite E4M3 magnitude
_E4M3_BIAS = 7
_E4M3_MIN_NORMAL = 2.0 ** -6
_E4M3_SUBNORMAL_QUANTUM = 2.0 ** -9   # (1/8) * 2^-6


def e4m3_value_table() -> np.ndarray:
    """Return the fp64 value of each of the 256 E4M3 codes (NaN for the 2 NaN codes).

    Built field by field from the format definition above, not from any library.
    """
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if (code >> 7) & 1 else 1.0
        exp_field = (code >> 3) & 0xF
        man = code & 0x7
        if exp_field == 0xF and man == 0x7:
            vals[code] = np.nan
        elif exp_field == 0:
            vals[code] = sign * (man / 8.0) * _E4M3_MIN_NORMAL
        else:
            vals[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp_field - _E4M3_BIAS)
    return vals


_TABLE = e4m3_value_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode uint8 E4M3 codes to fp64 values."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def _binade(a: np.ndarray) -> np.ndarray:
    """Exact floor(log2(a)) for a > 0 (0 for a == 0), via frexp: a = m * 2^ex, m in [0.5, 1)."""
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    return (ex - 1).astype(np.float64)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Encode finite values to E4M3 codes with round-to-nearest-even and satfinite.

    The magnitude is rounded on the grid that holds it: spacing 2^(e-3) in the
    normal binade [2^e, 2^(e+1)), spacing 2^-9 below 2^-6.  ``np.rint`` rounds a
    half-way quotient to the even integer, which is the even mantissa code.
    Magnitudes above 448 saturate to 448.  The sign bit is copied from x, so -0.0
    and negatives that round to zero give code 0x80.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode: non-finite input")
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    a = np.minimum(a, E4M3_MAX)                       # satfinite
    # spacing of the E4M3 grid around a
    e = _binade(a)
    e = np.maximum(e, -6.0)                           # below 2^-6 the spacing is constant
    quantum = np.where(a >= _E4M3_MIN_NORMAL, 2.0 ** (e - 3), _E4M3_SUBNORMAL_QUANTUM)
    v = np.rint(a / quantum) * quantum                # RNE onto the grid (exact in fp64)
    v = np.minimum(v, E4M3_MAX)                       # 448 is on the grid: a <= 448 never rounds past it
    # fields of the rounded magnitude
    is_normal = v >= _E4M3_MIN_NORMAL
    ve = _binade(np.where(is_normal, v, 1.0))
    man_norm = np.rint(v / 2.0 ** ve * 8.0 - 8.0)
    code_norm = ((ve + _E4M3_BIAS).astype(np.int64) << 3) | man_norm.astype(np.int64)
    code_sub = np.rint(v / _E4M3_SUBNORMAL_QUANTUM).astype(np.int64)
    mag = np.where(is_normal, code_norm, code_sub).astype(np.uint8)
    return (mag | sign).astype(np.uint8)


def quantize_rows(x_rows: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-row absmax FP8 quantisation.

    ``x_rows``: [rows, row_len] values exactly representable in fp32 (bf16 or fp32
    sources).  Returns ``(codes uint8 [rows, row_len], scale fp32 [rows])`` with
    ``scale = fp32(absmax)/448`` and ``codes = encode(fp32(x)/scale)``, both
    divisions in IEEE fp32 (numpy float32 division is correctly rounded).
    """
    x32 = np.asarray(x_rows, dtype=np.float32)
    if x32.ndim != 2:
        raise ValueError("quantize_rows expects a 2-D array")
    absmax = np.max(np.abs(x32), axis=1)
    scale = np.where(absmax > 0, absmax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (x32 / scale[:, None]).astype(np.float32)
    return e4m3_encode(scaled), scale


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact fp64 value of bf16 bit patterns (uint16): the bits are the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)
