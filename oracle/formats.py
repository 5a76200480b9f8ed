"""Number formats used by the compressed caches -- plain reference codecs.

TEST INFRASTRUCTURE ONLY.  This module is part of the CPU oracle: it may be
imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, never by the
library itself.

Sources
-------
* FP8 KV storage: "DeepSeek V4 1M context window agent efficient inference"
  (ai-papers.net), section "ハイブリッドアテンションの仕組み": most KV entries
  are stored in FP8 and the Lightning Indexer runs in FP4.
* FP4 packing: "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソース
  モデル" (studioglobal.ai), section "FP4/FP8混合精度": FP4 (MXFP4) values are
  packed two per byte.

The pages name the formats but not their bit layouts; the layouts below are
the OCP 8-bit (E4M3, "FN" variant: no infinities, one NaN pattern per sign)
and OCP MX 4-bit (E2M1) definitions, written out from the bit fields.

Every function works on numpy arrays and is exact: decoding produces float64
values, encoding rounds an exactly-known value (float64) to nearest-even.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0          # largest finite E4M3 magnitude: 1.75 * 2**8
E4M3_NAN = 0x7F           # S.1111.111 is NaN in the FN variant

# --------------------------------------------------------------------------
# E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
# --------------------------------------------------------------------------


def e4m3_decode(codes) -> np.ndarray:
    """Decode E4M3 bytes to float64.

    Exponent field 0 is subnormal: (m/8) * 2**-6.  Otherwise
    (1 + m/8) * 2**(e-7).  Pattern x.1111.111 decodes to NaN.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    out = sign * mag
    return np.where((c & 0x7F) == E4M3_NAN, np.nan, out)


def e4m3_encode(values) -> np.ndarray:
    """Round values (float64, exact) to E4M3, nearest-even, saturating at +-448.

    Saturation ("satfinite") maps every finite magnitude >= 448 to 448.  The
    rounding is done on the exact binary value: for a normal result the value
    is scaled so that its significand occupies [8, 16) units of the last place
    and rounded half-to-even; subnormals use a fixed unit of 2**-9.
    """
    v = np.asarray(values, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("e4m3_encode: NaN input")
    sign = (np.signbit(v)).astype(np.int64) << 7
    a = np.abs(v)
    code = np.zeros(a.shape, dtype=np.int64)

    sat = a >= E4M3_MAX
    sub = a < 2.0 ** -6
    nor = ~sat & ~sub

    # subnormal range: unit 2**-9, n in [0, 8]; n == 8 is the smallest normal
    # (exponent field 1, mantissa 0) whose code is also 8.
    n_sub = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)
    code[sub] = n_sub

    # normal range: a = f * 2**k with f in [0.5, 1); exponent of the leading
    # bit is k-1.  Significand in units of 2**(e-3) lies in [8, 16).
    f, k = np.frexp(a[nor])
    e = k - 1
    n = np.rint(np.ldexp(f, 4)).astype(np.int64)   # f*16 in [8, 16] after rounding
    carry = n == 16
    n = np.where(carry, 8, n)
    e = np.where(carry, e + 1, e)
    code[nor] = ((e + 7) << 3) | (n - 8)

    code[sat] = 0x7E
    return (code | sign).astype(np.uint8)


# --------------------------------------------------------------------------
# E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
# --------------------------------------------------------------------------


def e2m1_decode(nibbles) -> np.ndarray:
    """Decode 4-bit E2M1 codes (0..15) to float64.

    Exponent field 0 is subnormal: m * 0.5.  Otherwise (1 + m/2) * 2**(e-1).
    The magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
    """
    c = np.asarray(nibbles).astype(np.int64)
    if ((c < 0) | (c > 15)).any():
        raise ValueError("e2m1_decode: codes must be 4-bit")
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e - 1.0))
    return sign * mag


def e2m1_unpack(packed) -> np.ndarray:
    """Split packed E2M1 bytes [..., d/2] into codes [..., d].

    Element 2j is the low nibble of byte j and element 2j+1 the high nibble.
    """
    p = np.asarray(packed, dtype=np.uint8)
    lo = p & 0x0F
    hi = p >> 4
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# E2M1 magnitudes in code order (codes 0..7; bit 3 is the sign)
E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def e2m1_encode(values) -> np.ndarray:
    """Round exactly-known values (float64) to E2M1 codes (0..15).

    Nearest value of the grid, ties to the code with an even mantissa bit
    (the even code), magnitudes above 6 saturate to 6.  The sign is kept,
    so a negative value that rounds to zero gives the code of -0 (0x8).
    """
    v = np.asarray(values, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("e2m1_encode: NaN")
    mag = np.minimum(np.abs(v), 6.0)
    grid = np.asarray(E2M1_GRID)
    lo = np.clip(np.searchsorted(grid, mag, side="right") - 1, 0, 7)   # grid[lo] <= mag
    hi = np.minimum(lo + 1, 7)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    up = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(up, hi, lo).astype(np.uint8)
    sign = np.where(np.signbit(v), 0x8, 0x0).astype(np.uint8)
    return (code | sign).astype(np.uint8)


def e2m1_pack(codes) -> np.ndarray:
    """Pack codes [..., d] (d even) two per byte: element 2j in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


# --------------------------------------------------------------------------
# E8M0: an 8-bit power-of-two scale, 2**(code - 127); 0xFF is NaN.
# --------------------------------------------------------------------------


def e8m0_decode(codes) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64)
    return np.where(c == 0xFF, np.nan, np.exp2((c - 127).astype(np.float64)))


# --------------------------------------------------------------------------
# MXFP4: blocks of 32 elements, E2M1 elements and one E8M0 scale per block.
# --------------------------------------------------------------------------
MX_BLOCK = 32


def mxfp4_quantize(x):
    """Quantise fp32 values [rows, cols] (cols a multiple of 32) to MXFP4.

    Source: "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
    (studioglobal.ai), section "FP4/FP8混合精度" -- FP4 values are MXFP4,
    packed two per byte.  The pages give no rounding rule; this is the OCP
    microscaling conversion written out: per block of 32 consecutive
    elements, X = floor(log2(max|v|)) - 2 (2 being the exponent of the
    largest E2M1 value, 6 = 1.5 * 2**2), at least -127 (an all-zero block
    takes -127); scale = 2**X stored as the E8M0 code X + 127; each element
    v / 2**X (exact) rounded by e2m1_encode.

    Returns (packed codes u8 [rows, cols/2], scale codes u8 [rows, cols/32]).
    """
    v = np.asarray(x, dtype=np.float32).astype(np.float64)
    if v.ndim != 2 or v.shape[1] % MX_BLOCK:
        raise ValueError("mxfp4_quantize: expects [rows, cols] with cols a multiple of 32")
    rows, cols = v.shape
    blocks = v.reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    _, e = np.frexp(amax)                      # amax = f * 2**e, f in [0.5, 1): floor(log2) = e - 1
    X = np.where(amax > 0, e - 1 - 2, -127)
    X = np.maximum(X, -127).astype(np.int64)
    r = blocks / np.exp2(X.astype(np.float64))[..., None]
    codes = e2m1_encode(r).reshape(rows, cols)
    return e2m1_pack(codes), (X + 127).astype(np.uint8)


# --------------------------------------------------------------------------
# bf16: the top half of an IEEE binary32.
# --------------------------------------------------------------------------


def bf16_decode(bits) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float64 exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):       # NaN payloads stay NaN
        return b.view(np.float32).astype(np.float64)
