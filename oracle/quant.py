"""NVFP4 quantizer, dequantizer and scale-factor tile map (oracle side).

What the pages fix
------------------
* NVFP4 = E2M1 elements, one E4M3 block scale per 16 elements, plus an FP32 global scale
  ("May 24, 2026 — Session Start Plan", section 1 "NVFP4-0: Verify FP4 Primitives").
* The global scale ("gsa", global_scale_a) comes from the amax of the whole tensor, on the
  GPU, into a GPU buffer that the GEMM reads (commit log of dsv4/kernels/cuda: the
  "Two-kernel approach" fix, kernels amax_gsa.cu then quantize_nvfp4_from_buffer).
* The element codes are computed against the FP8-round-tripped block scale, because the
  dequantizer reads the FP8 byte back (same commit log, the "CRITICAL: quantize must use the
  FP8-round-tripped block scale" commit; the raw scale was the cause of cos 0.925).

Readings where the pages are silent
-----------------------------------
* gs = 448 * 6 / amax: the largest block scale lands on E4M3's maximum.  If the quotient is
  not a finite positive float32 (amax 0, inf or NaN) gs = 1.
* FP32 operation order, one rounding per operation (numpy float32 arithmetic):
    s = (a_b / 6) * gs ;  sf = E4M3(s) ;  d = decode(sf) ;  r = gs / d ;  code_i = E2M1(x_i * r)
  A block whose decoded scale is 0 gets all-zero codes; a zero element encodes as a (signed)
  zero without the multiply, so 0 * r stays 0 when gs / d overflows for extreme inputs.
* Dequantized value = E2M1(code) * d / gs.

Scale-factor tile layout
------------------------
Block scales are stored tiled as the block-scaled tensor-core MMA consumes them: the
(rows x cols/16) scale matrix is cut into 128-row x 4-column atoms of 512 bytes, atoms
row-major over (rows/128, cols/64); inside an atom, scale (r, c) sits at byte
(r % 32) * 16 + (r // 32) * 4 + c.  The pages only say the layout is handled by CuTe's
block-scaled layout utilities ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section
"Reference Files" and table "Key Differences"), so this reading is ours.
"""

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, pack_nibbles, unpack_nibbles

BLOCK = 16
GS_NUMERATOR = np.float32(448.0 * 6.0)  # E4M3 max times E2M1 max


def global_scale(x):
    """FP32 global scale from the amax of the whole tensor: gs = 2688 / max|x| (float32).

    Falls back to 1.0 when the quotient is not a finite positive number.
    """
    a = np.max(np.abs(np.asarray(x, dtype=np.float32))) if np.size(x) else np.float32(0)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        gs = np.float32(GS_NUMERATOR / np.float32(a))
    if not (np.isfinite(gs) and gs > 0):
        gs = np.float32(1.0)
    return np.float32(gs)


def scale_from_amax(amax):
    """FP32 global scale from a GIVEN amax: 2688 / amax, 1.0 when that is not a finite positive
    float32.  The rule of :func:`global_scale`, with the amax supplied rather than taken from the
    tensor being quantized.

    Reading for the intermediate h (the pages derive every activation's global scale from its
    amax on the GPU — commit log of dsv4/kernels/cuda, the "Two-kernel approach" fix — but fuse
    h's re-quantization into the L1 epilogue, "May 24, 2026 — Session Start Plan", section 5
    "NVFP4-1.1", where the amax of all of h is not known when a tile is written): delayed
    scaling.  Call i quantizes h with scale_from_amax(amax of h in call i-1); a first call uses
    a given scale.
    """
    a = np.float32(amax)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        gs = np.float32(GS_NUMERATOR / a)
    if not (np.isfinite(gs) and gs > 0):
        gs = np.float32(1.0)
    return np.float32(gs)


def block_scale_clipping(x, gs):
    """How many 16-element block scales of ``x`` (rows, cols) the E4M3 format could not hold at
    global scale ``gs``: (saturated, underflowed).

    saturated   s = (a_b / 6) * gs exceeds 448, E4M3's largest value, and was clipped to it
                (the block's largest elements then saturate at E2M1's 6)
    underflowed a_b > 0 but s rounds to the E4M3 zero (s <= 2^-10), so every code of the
                block is 0
    s is the float32 value the quantizer computes (two roundings, as in :func:`quantize`).
    Parity note: the pages name no such count; it measures how well a static or delayed gs
    fits the data, the trade-off a fused epilogue makes.
    """
    x32 = np.asarray(x, dtype=np.float32)
    rows, cols = x32.shape
    blocks = x32.reshape(rows, cols // BLOCK, BLOCK)
    a_b = np.max(np.abs(blocks), axis=-1)
    s = ((a_b / np.float32(6.0)).astype(np.float32) * np.float32(gs)).astype(np.float32)
    saturated = int(np.count_nonzero(s > np.float32(448.0)))
    underflowed = int(np.count_nonzero((a_b > 0) & (e4m3_encode(s) & 0x7F == 0)))
    return saturated, underflowed


def quantize(x, gs):
    """Quantize a (rows, cols) array to NVFP4 with global scale ``gs`` (float32).

    Returns (codes uint8 (rows, cols) unpacked nibbles, sf uint8 (rows, cols/16) E4M3 bytes).
    Every arithmetic step is a single float32 operation in the order listed in the module
    docstring; the element codes use the decoded (round-tripped) block scale.
    """
    x32 = np.asarray(x, dtype=np.float32)
    rows, cols = x32.shape
    assert cols % BLOCK == 0
    gs = np.float32(gs)
    blocks = x32.reshape(rows, cols // BLOCK, BLOCK)
    a_b = np.max(np.abs(blocks), axis=-1)                      # exact
    s = (a_b / np.float32(6.0)).astype(np.float32) * gs        # two float32 roundings
    s = s.astype(np.float32)
    sf = e4m3_encode(s)
    d = e4m3_decode(sf).astype(np.float32)                     # exact (E4M3 fits float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        r = (gs / d).astype(np.float32)
        y = (blocks * r[..., None]).astype(np.float32)
    y = np.where(blocks == 0, blocks, y)  # 0 * r is 0 even when r overflowed to inf
    zero_blk = (d == 0)[..., None]
    y = np.where(zero_blk, np.float32(0.0), y)
    codes = e2m1_encode(y)
    codes = np.where(zero_blk, np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(rows, cols), sf


def quantize_raw_scale(x, gs):
    """The faulty variant the commit log describes: codes computed against the raw (not
    FP8-round-tripped) block scale.  Used only by a test that shows the two differ."""
    x32 = np.asarray(x, dtype=np.float32)
    rows, cols = x32.shape
    gs = np.float32(gs)
    blocks = x32.reshape(rows, cols // BLOCK, BLOCK)
    a_b = np.max(np.abs(blocks), axis=-1)
    s = ((a_b / np.float32(6.0)).astype(np.float32) * gs).astype(np.float32)
    sf = e4m3_encode(s)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        r = (gs / s).astype(np.float32)
        y = np.where((s == 0)[..., None], np.float32(0), (blocks * r[..., None]).astype(np.float32))
    return e2m1_encode(y).reshape(rows, cols), sf


def dequantize(codes, sf, gs):
    """float64 values E2M1(code) * decode(sf) / gs for unpacked codes (rows, cols)."""
    c = np.asarray(codes, dtype=np.uint8)
    rows, cols = c.shape
    d = e4m3_decode(sf).astype(np.float64)
    v = e2m1_decode(c).reshape(rows, cols // BLOCK, BLOCK) * d[..., None]
    return (v / np.float64(gs)).reshape(rows, cols)


def quantize_packed(x, gs):
    """quantize() with the codes packed two per byte: (rows, cols/2) and sf (rows, cols/16)."""
    codes, sf = quantize(x, gs)
    return pack_nibbles(codes), sf


def dequantize_packed(packed, sf, gs):
    return dequantize(unpack_nibbles(packed), sf, gs)


# ----------------------------------------------------------------------- tiled SF layout

def sf_tile_offset(r, c, n_sf_cols):
    """Byte offset of block scale (row r, scale column c) in the tiled layout.

    ``n_sf_cols`` = cols / 16 (a multiple of 4).  Atoms of 128 rows x 4 scale columns, 512 B,
    row-major over (row // 128, c // 4); inside an atom (r%32)*16 + ((r//32)%4)*4 + c%4.
    """
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    atoms_per_row = n_sf_cols // 4
    atom = (r // 128) * atoms_per_row + (c // 4)
    inner = (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)
    return atom * 512 + inner


def tile_sf(sf):
    """(rows, n) logical scale matrix -> flat tiled bytes; rows % 128 == 0, n % 4 == 0."""
    sf = np.asarray(sf, dtype=np.uint8)
    rows, n = sf.shape
    assert rows % 128 == 0 and n % 4 == 0
    out = np.zeros(rows * n, dtype=np.uint8)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(n), indexing="ij")
    out[sf_tile_offset(rr, cc, n)] = sf
    return out


def untile_sf(flat, rows, n):
    """Inverse of :func:`tile_sf`."""
    flat = np.asarray(flat, dtype=np.uint8).reshape(-1)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(n), indexing="ij")
    return flat[sf_tile_offset(rr, cc, n)]
