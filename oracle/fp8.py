"""fp64 reference for the 8-bit (E4M3) latent cache: rounding, codes, per-token scales.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): the library never imports this.

Source. The softved page "Introduction to MLA vs. KV Cache in Large Language Models",
section "Practical Implementation Tips for MLA in LLM Serving", advises quantising the
cache on top of the latent compression; it fixes no format. The readings taken here:

  * Element format: E4M3 of the OCP 8-bit floating point specification (OFP8): one
    sign bit, four exponent bits with bias 7, three mantissa bits; exponent field 0
    holds the subnormals m * 2^-9 (m = 0..7); no infinities; S.1111.111 is NaN, so
    the largest finite magnitude is 1.75 * 2^8 = 448.
  * Rounding: to nearest, ties to the even code, saturating: a magnitude that would
    round above 448 becomes 448 (no NaN is ever produced from a finite input). The
    sign of a result that rounds to zero is kept (0x80 is -0).
  * Scale: one power of two 2^k per cached row (token), shared by its latent and its
    rope key, stored as the biased byte e = k + 127 (the E8M0 convention). k is the
    smallest integer in [-126, 7] with max_i |x_i| <= 448 * 2^k; a row larger than
    448 * 2^7 keeps k = 7 and saturates. The code of x_i is round(x_i * 2^-k); the row
    dequantises to code * 2^k exactly.

Everything is float64; scaling by powers of two is exact, so the rounding decision is
made on the exact value x_i * 2^-k.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_STEP = 2.0 ** -9
SCALE_K_MIN, SCALE_K_MAX = -126, 7
SCALE_BIAS = 127


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448; float64 out."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # the spacing of the E4M3 grid around |x|: 2^(E-3) in binade [2^E, 2^(E+1)), E >= -6,
    # and the subnormal step 2^-9 below 2^-6
    _, e = np.frexp(np.where(a > 0, a, 1.0))          # a = f * 2^e, f in [0.5, 1)
    E = e.astype(np.int64) - 1
    quantum = np.where(a >= E4M3_MIN_NORMAL, np.ldexp(1.0, E - 3), E4M3_SUBNORMAL_STEP)
    r = np.rint(a / quantum) * quantum                 # np.rint: halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code byte (0x7F and 0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(ef == 0, m * E4M3_SUBNORMAL_STEP, np.ldexp(1.0 + m / 8.0, ef - 7))
    mag = np.where((ef == 0xF) & (m == 0x7), np.nan, mag)
    return s * mag


def e4m3_encode(v) -> np.ndarray:
    """Code byte of each E4M3 value (values must already lie on the grid)."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.int64) << 7
    a = np.abs(v)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    E = e.astype(np.int64) - 1
    normal = a >= E4M3_MIN_NORMAL
    ef = np.where(normal, E + 7, 0)
    m = np.where(normal, np.ldexp(a, -E) * 8.0 - 8.0, a / E4M3_SUBNORMAL_STEP)
    mi = np.rint(m).astype(np.int64)
    if np.any(np.abs(m - mi) > 0) or np.any(ef > 15) or np.any((ef == 15) & (mi == 7)):
        raise ValueError("value not on the E4M3 grid")
    return (sign | (ef << 3) | mi).astype(np.uint8)


def row_scale_exponent(rows) -> np.ndarray:
    """k per row: the smallest integer in [-126, 7] with max|x| <= 448 * 2^k."""
    x = np.asarray(rows, dtype=np.float64)
    amax = np.max(np.abs(x), axis=-1) if x.shape[-1] else np.zeros(x.shape[:-1])
    k = np.full(amax.shape, SCALE_K_MIN, dtype=np.int64)
    # raise k one step at a time while the row still overflows the code range
    for _ in range(SCALE_K_MAX - SCALE_K_MIN):
        over = (amax > np.ldexp(E4M3_MAX, k)) & (k < SCALE_K_MAX)
        if not over.any():
            break
        k = k + over
    return k


def quantise_rows(rows):
    """(codes uint8 [..., n], scale bytes uint8 [...]) of cache rows [..., n]."""
    x = np.asarray(rows, dtype=np.float64)
    k = row_scale_exponent(x)
    codes = e4m3_encode(e4m3_round(np.ldexp(x, -k[..., None])))
    return codes, (k + SCALE_BIAS).astype(np.uint8)


def dequantise_rows(codes, scale_bytes) -> np.ndarray:
    """The float64 rows the codes stand for: code * 2^(e - 127), exact (the code's value
    read from the table of all 256 decoded codes)."""
    k = np.asarray(scale_bytes, dtype=np.int64) - SCALE_BIAS
    table = e4m3_decode(np.arange(256, dtype=np.uint8))
    return np.ldexp(table[np.asarray(codes, dtype=np.uint8)], k[..., None])
