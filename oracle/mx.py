"""MXFP4 quantizer and dequantizer (oracle side): the format the pages contrast with NVFP4.

Test infrastructure, not product: only the test suite may use it.

What the pages fix
------------------
* MXFP4 has 32-element blocks with UE8M0 (power-of-two) scales, where NVFP4 has 16-element
  blocks with E4M3 scales ("May 24, 2026 — Session Start Plan", section 1 "NVFP4-0", items
  NVFP4-0.1 and NVFP4-0.4).  The elements are E2M1 in both.

Readings where the pages are silent (the OCP Microscaling (MX) v1.0 definition)
-----------------------------------------------------------------------------
* Shared scale of a block: X = 2^e with e = floor(log2(max|x_i|)) - 2, where 2 is the exponent of
  E2M1's largest normal value (6 = 1.5 * 2^2).  e is clamped to the UE8M0 range [-127, 127]; an
  all-zero block takes e = -127.  The scale byte is e + 127 (255 is NaN, never produced).
* Elements: code_i = E2M1_RN_even(x_i / X), saturating: a block's amax lies in [4X, 8X), so
  values above 6X are clipped to +-6 (the format's known clipping).
* Dequantized value = E2M1(code) * 2^(byte - 127).  No global scale: the power-of-two block
  scale spans the range by itself.
* x / X is exact in float64 (a power-of-two divisor) for every finite bf16 or float32 input.
"""

import numpy as np

from .formats import e2m1_decode, e2m1_encode

MX_BLOCK = 32
E2M1_EMAX = 2      # exponent of the largest E2M1 normal value, 6 = 1.5 * 2^2
E8M0_BIAS = 127


def e8m0_decode(b):
    """UE8M0 byte -> float64: 2^(b - 127) for b < 255, NaN for 255."""
    b = np.asarray(b, dtype=np.int64)
    v = np.ldexp(1.0, b - E8M0_BIAS)
    return np.where(b == 255, np.nan, v)


def block_exponent(amax):
    """e = floor(log2(amax)) - 2, clamped to [-127, 127]; -127 for amax == 0.

    floor(log2) is taken exactly from the binary exponent (frexp: amax = m * 2^k, m in [0.5, 1),
    so floor(log2(amax)) = k - 1)."""
    a = np.asarray(amax, dtype=np.float64)
    _, k = np.frexp(a)
    e = (k - 1) - E2M1_EMAX
    e = np.where(a > 0, e, -E8M0_BIAS)
    return np.clip(e, -E8M0_BIAS, E8M0_BIAS).astype(np.int64)


def quantize_mxfp4(x):
    """(rows, cols) float -> (codes uint8 (rows, cols) unpacked E2M1, scale bytes uint8
    (rows, cols / 32)).  cols % 32 == 0."""
    x64 = np.asarray(x, dtype=np.float64)
    rows, cols = x64.shape
    assert cols % MX_BLOCK == 0
    blocks = x64.reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    e = block_exponent(np.max(np.abs(blocks), axis=-1))
    y = np.ldexp(blocks, -e[..., None])          # exact: x / 2^e
    codes = e2m1_encode(y)                       # RN-even, saturating at +-6
    return codes.reshape(rows, cols).astype(np.uint8), (e + E8M0_BIAS).astype(np.uint8)


def dequantize_mxfp4(codes, scales):
    """float64 values E2M1(code) * 2^(scale - 127) for unpacked codes (rows, cols)."""
    c = np.asarray(codes, dtype=np.uint8)
    rows, cols = c.shape
    v = e2m1_decode(c).reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    return (v * e8m0_decode(scales)[..., None]).reshape(rows, cols)
