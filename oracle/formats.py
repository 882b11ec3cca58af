"""E2M1 (FP4) and E4M3 (FP8) codecs, written from the format definitions.

Sources
-------
* E2M1 magnitudes and bit layout: commit log of ``dsv4/kernels/cuda`` in nvfp4-megamoe-kernel,
  the indexer E2M1-decode fix ("E2M1 encoding (bias=1)": exponent 0 subnormal gives 0 and 0.5,
  exponents 1..3 give 1, 1.5, 2, 3, 4, 6; a sign bit on top).
* E4M3 as the NVFP4 block-scale type (not UE8M0): "May 24, 2026 — Session Start Plan",
  section 1 "NVFP4-0: Verify FP4 Primitives".  The pages name the type only, so the bit
  semantics follow the OCP 8-bit floating point definition: bias 7, no infinities,
  S.1111.111 is NaN, largest finite 448, subnormals m * 2^-9.
* Two FP4 codes per byte (``float4_e2m1fn_x2``), same section.  Element 2j sits in the low
  nibble and element 2j+1 in the high nibble (the pages only name the packed type).

Rounding for both encoders is round-to-nearest, ties to the even mantissa, with saturation
to the largest finite magnitude (``satfinite``).  The sign of a value that rounds to zero is
kept (-0 encodes as 0x8 / 0x80).
"""

import numpy as np

# Magnitudes of the eight E2M1 codes 0b000..0b111 (sign is bit 3).
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


# --------------------------------------------------------------------------- E2M1

def e2m1_decode(codes):
    """Decode 4-bit E2M1 codes (uint8 array, values 0..15) to float64.

    Bit 3 is the sign; bits 2..0 index ``E2M1_MAGNITUDES`` (exponent bias 1, exponent 0 is
    subnormal with value 0.5 * mantissa).
    """
    c = np.asarray(codes, dtype=np.uint8)
    mag = np.asarray(E2M1_MAGNITUDES, dtype=np.float64)[c & 0x7]
    return np.where((c & 0x8) != 0, -mag, mag)


def _quantum_e2m1(a):
    """Spacing of the E2M1 grid at magnitude ``a`` (float64 array, a < 6).

    Exponent field 0 (subnormal) and 1 share the spacing 0.5; each further binade doubles it.
    ``frexp`` gives a = f * 2^e with f in [0.5, 1), so floor(log2 a) = e - 1 exactly.
    """
    _, e = np.frexp(a)
    unbiased = np.maximum(e - 1, 0)  # binade of a, clamped at the subnormal binade
    return np.ldexp(1.0, unbiased - 1)  # one mantissa bit


def e2m1_encode(y):
    """Encode float32/float64 values to E2M1 codes (uint8), RN-even, satfinite.

    |y| >= 6 gives 6 (saturation; also covers +-inf).  NaN is not a valid input.
    """
    y = np.asarray(y, dtype=np.float64)
    if np.isnan(y).any():
        raise ValueError("e2m1_encode: NaN input")
    a = np.abs(y)
    sat = a >= E2M1_MAX
    a_c = np.where(sat, 0.0, a)
    q = _quantum_e2m1(np.where(a_c == 0.0, 1.0, a_c))
    k = np.rint(a_c / q)  # np.rint rounds half to even; k even <=> mantissa bit even
    val = np.where(sat, E2M1_MAX, k * q)
    val = np.minimum(val, E2M1_MAX)
    table = np.asarray(E2M1_MAGNITUDES)
    idx = np.searchsorted(table, val)
    assert np.all(table[np.minimum(idx, 7)] == val), "value off the E2M1 grid"
    code = idx.astype(np.uint8)
    return np.where(np.signbit(y), code | 0x8, code).astype(np.uint8)


def pack_nibbles(codes):
    """Pack E2M1 codes along the last axis, two per byte: element 2j low nibble, 2j+1 high."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed):
    """Inverse of :func:`pack_nibbles`."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# --------------------------------------------------------------------------- E4M3

def e4m3_decode(b):
    """Decode E4M3 bytes to float64 (bias 7; exponent 0 subnormal m*2^-9; 0x7F/0xFF NaN)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    sub = m * 2.0 ** -9
    val = sign * np.where(e == 0, sub, normal)
    return np.where((b & 0x7F) == 0x7F, np.nan, val)


def e4m3_encode(v):
    """Encode float32/float64 values to E4M3 bytes, RN-even, satfinite.

    |v| >= 448 (including infinity) gives 448; NaN gives 0x7F.
    """
    v = np.asarray(v, dtype=np.float64)
    nan = np.isnan(v)
    a = np.abs(np.where(nan, 0.0, v))
    sat = a >= E4M3_MAX
    a_c = np.where(sat, 0.0, a)
    _, e = np.frexp(np.where(a_c == 0.0, 1.0, a_c))
    unbiased = np.maximum(e - 1, -6)  # binade, clamped at the subnormal binade 2^-6
    q = np.ldexp(1.0, unbiased - 3)  # three mantissa bits
    val = np.rint(a_c / q) * q
    val = np.where(sat, E4M3_MAX, np.minimum(val, E4M3_MAX))
    # value -> fields
    _, e2 = np.frexp(np.where(val == 0.0, 1.0, val))
    ebin = e2 - 1
    is_norm = val >= 2.0 ** -6
    exp_field = np.where(is_norm, ebin + 7, 0)
    mant = np.where(is_norm, np.ldexp(val, -ebin) * 8.0 - 8.0, val / 2.0 ** -9)
    assert np.all(mant == np.rint(mant)), "value off the E4M3 grid"
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(np.signbit(v) & ~nan, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)
