"""Pins for the oracle's NVFP4 quantizer, dequantizer and scale tile map (CPU only)."""

import numpy as np
import pytest

from oracle import formats as F
from oracle import quant as Q


def test_global_scale_closed_forms():
    assert Q.global_scale(np.array([2688.0, -1.0])) == 1.0
    assert Q.global_scale(np.array([0.5, -1.0])) == 2688.0
    assert Q.global_scale(np.zeros(16)) == 1.0           # amax 0 -> fallback
    assert Q.global_scale(np.array([np.inf])) == 1.0     # 2688/inf = 0 -> fallback
    assert Q.global_scale(np.array([3.0])) == np.float32(2688.0) / np.float32(3.0)


def test_dequantize_hand_example():
    # code 0b0101 = 3.0, scale byte 0x38 = 1.0 (exponent field 7, mantissa 0), gs = 2 -> 1.5
    codes = np.array([[5] + [0] * 15], dtype=np.uint8)
    sf = np.array([[0x38]], dtype=np.uint8)
    assert Q.dequantize(codes, sf, 2.0)[0, 0] == 1.5
    # code 0b1111 = -6, scale byte 0x40 = 2.0, gs = 0.5 -> -24
    codes[0, 1] = 15
    sf[0, 0] = 0x40
    assert Q.dequantize(codes, sf, 0.5)[0, 1] == -24.0


@pytest.mark.parametrize("sf_byte", [0x08, 0x30, 0x38, 0x39, 0x4B, 0x66, 0x7E, 0x05])
@pytest.mark.parametrize("gs", [1.0, 64.0, 2.0 ** -7])
def test_round_trip_on_grid_blocks(sf_byte, gs):
    """A block whose values are E2M1 grid points times d/gs, with one element at +-6, must
    quantize back to the same codes and the same scale byte."""
    rng = np.random.default_rng(sf_byte)
    d = F.e4m3_decode(np.uint8(sf_byte))
    codes = rng.integers(0, 16, size=(4, 16)).astype(np.uint8)
    codes[:, 3] = rng.choice([7, 15], size=4)  # amax element = 6 * d / gs
    x = (F.e2m1_decode(codes) * d / gs).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), F.e2m1_decode(codes) * d / gs)  # exact
    c2, sf2 = Q.quantize(x, np.float32(gs))
    assert np.all(sf2 == sf_byte)
    # +-0 decode alike; compare values, and the codes of nonzero elements bit-exactly
    nz = (codes & 7) != 0
    assert np.array_equal(c2[nz], codes[nz])
    assert np.all((c2[~nz] & 7) == 0)


def test_error_bound_per_element():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 256)).astype(np.float32) * np.float32(3.0)
    gs = Q.global_scale(x)
    codes, sf = Q.quantize(x, gs)
    xh = Q.dequantize(codes, sf, gs)
    d = F.e4m3_decode(sf).repeat(16, axis=1)
    y = np.abs(x.astype(np.float64)) * gs / d
    spacing = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    bound = 0.5 * spacing * d / gs * (1 + 1e-6) + 1e-30
    # the FP8 scale can round down by half an E4M3 step (1/16), so y reaches 6 * 17/16 at most;
    # those elements saturate to 6, still within half the top spacing (2)
    assert y.max() <= 6 * 17 / 16 * (1 + 1e-6)
    assert (y > 6).any()
    assert np.all(np.abs(x - xh) <= bound)


def test_round_tripped_scale_differs_from_raw_scale():
    """The commit log's bug: codes against the raw (pre-FP8) scale differ from codes against
    the decoded FP8 byte; here s = 1.0625 rounds to the byte for 1.0 (tie to even)."""
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0] = 6.375          # block amax: s = 6.375 / 6 = 1.0625 -> E4M3 1.0
    x[0, 1] = 2.6            # /1.0 -> 2.6 -> code 3.0 ; /1.0625 -> 2.447 -> code 2.0
    good, sf = Q.quantize(x, np.float32(1.0))
    bad, sf_bad = Q.quantize_raw_scale(x, np.float32(1.0))
    assert sf[0, 0] == sf_bad[0, 0] == 0x38
    assert F.e2m1_decode(good[0, 1]) == 3.0
    assert F.e2m1_decode(bad[0, 1]) == 2.0


def _cos(a, b):
    a = a.ravel().astype(np.float64)
    b = b.ravel().astype(np.float64)
    return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))


def test_cosine_sanity_range_and_raw_scale_is_worse():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((256, 1024)).astype(np.float32)
    gs = Q.global_scale(x)
    c, sf = Q.quantize(x, gs)
    cos_good = _cos(x, Q.dequantize(c, sf, gs))
    cb, sfb = Q.quantize_raw_scale(x, gs)
    cos_bad = _cos(x, Q.dequantize(cb, sfb, gs))
    assert 0.99 <= cos_good <= 0.9975
    assert cos_bad < cos_good


def test_all_zero_block_and_tiny_block():
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 16] = 1e-30  # block 1: s underflows E4M3 -> scale 0 -> zero codes
    x[0, 17] = 5.0
    x[0, 0] = 0.0
    gs = np.float32(1.0)
    c, sf = Q.quantize(x, gs)
    assert sf[0, 0] == 0 and np.all(c[0, :16] == 0)
    assert sf[0, 1] != 0


def test_sf_tile_offsets_hand_worked():
    # K = 128 -> 8 scale columns -> 2 atoms per 128-row block
    n = 8
    assert Q.sf_tile_offset(0, 0, n) == 0
    assert Q.sf_tile_offset(1, 0, n) == 16
    assert Q.sf_tile_offset(32, 0, n) == 4
    assert Q.sf_tile_offset(33, 5, n) == 512 + 16 + 4 + 1
    assert Q.sf_tile_offset(127, 3, n) == 31 * 16 + 3 * 4 + 3
    assert Q.sf_tile_offset(128, 0, n) == 2 * 512
    assert Q.sf_tile_offset(200, 7, n) == (1 * 2 + 1) * 512 + (200 % 32) * 16 + ((200 // 32) % 4) * 4 + 3


def test_sf_tile_is_bijection_and_inverse():
    rows, n = 256, 12
    rng = np.random.default_rng(5)
    sf = rng.integers(0, 256, size=(rows, n)).astype(np.uint8)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(n), indexing="ij")
    off = Q.sf_tile_offset(rr, cc, n).ravel()
    assert len(np.unique(off)) == rows * n and off.min() == 0 and off.max() == rows * n - 1
    assert np.array_equal(Q.untile_sf(Q.tile_sf(sf), rows, n), sf)
    # one 128x4 atom is 512 contiguous bytes
    t = Q.tile_sf(sf)
    assert np.array_equal(np.sort(t[:512]), np.sort(sf[:128, :4].ravel()))


def test_pack_roundtrip_quantize_packed():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    gs = Q.global_scale(x)
    p, sf = Q.quantize_packed(x, gs)
    c, sf2 = Q.quantize(x, gs)
    assert p.shape == (8, 32) and np.array_equal(sf, sf2)
    assert np.array_equal(Q.dequantize_packed(p, sf, gs), Q.dequantize(c, sf, gs))


# --------------------------------------------- delayed scale of the intermediate, clipping counts

def test_scale_from_amax_closed_forms():
    assert Q.scale_from_amax(2688.0) == 1.0
    assert Q.scale_from_amax(1.0) == 2688.0
    assert Q.scale_from_amax(0.5) == 5376.0
    assert Q.scale_from_amax(3.0) == np.float32(2688.0) / np.float32(3.0)
    for bad in (0.0, np.inf, np.nan, -1.0):
        assert Q.scale_from_amax(bad) == 1.0


def test_delayed_scale_from_the_same_data_is_the_dynamic_scale():
    """Quantizing h with the scale derived from its own amax (delayed scaling on an unchanged
    batch) gives exactly the dynamic quantization."""
    rng = np.random.default_rng(11)
    for scale in (1e-4, 0.3, 7.0, 5e3):
        h = (rng.standard_normal((32, 128)) * scale).astype(np.float32)
        amax = np.max(np.abs(h))
        assert Q.scale_from_amax(amax) == Q.global_scale(h)
        c1, s1 = Q.quantize(h, Q.scale_from_amax(amax))
        c2, s2 = Q.quantize(h, Q.global_scale(h))
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_block_scale_clipping_hand_cases():
    """gs = 1, one block per row.  The E4M3 largest value is 448 and its smallest subnormal 2^-9;
    s = a_b / 6, rounded to float32."""
    rows = np.zeros((6, 16), np.float32)
    rows[0, 3] = 6 * 448          # s = 448 exactly: held
    rows[1, 3] = 6 * 449          # s = 449 > 448: saturated
    rows[2, 5] = 6 * 2.0 ** -10   # s = 2^-10: the tie between 0 and 2^-9 goes to 0: underflowed
    rows[3, 5] = 6 * 2.0 ** -9    # s = 2^-9, the smallest subnormal: held
    rows[4, 0] = -6 * 2.0 ** -12  # s = 2^-12: underflowed (the sign does not matter)
    # row 5: all zero, neither
    assert Q.block_scale_clipping(rows, np.float32(1.0)) == (1, 2)
    # the same data at gs = 2^-3 brings row 1 into range and pushes row 3 under (s = 2^-12)
    assert Q.block_scale_clipping(rows, np.float32(0.125)) == (0, 3)


def test_block_scale_clipping_agrees_with_the_quantizer():
    """An underflowed block is exactly a nonzero block whose codes all come out 0; a saturated
    block has scale byte 0x7E (448) and its largest element dequantizes to 6 * 448 / gs, below
    its true magnitude."""
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-12, 8, (64, 1)))).astype(np.float32)
    gs = np.float32(64.0)
    sat, under = Q.block_scale_clipping(x, gs)
    codes, sf = Q.quantize(x, gs)
    blocks = x.reshape(64, 16, 16)
    nz = np.max(np.abs(blocks), axis=-1) > 0
    zero_codes = np.all((codes.reshape(64, 16, 16) & 7) == 0, axis=-1)
    assert under == int(np.count_nonzero(nz & zero_codes)) and under > 0
    s = ((np.max(np.abs(blocks), -1) / np.float32(6)).astype(np.float32) * gs).astype(np.float32)
    big = s > 448
    assert sat == int(np.count_nonzero(big)) and sat > 0
    assert np.all(sf[big] == 0x7E)
    xh = Q.dequantize(codes, sf, gs).reshape(64, 16, 16)
    amax_i = np.argmax(np.abs(blocks), axis=-1)
    top = np.take_along_axis(np.abs(xh), amax_i[..., None], -1)[..., 0]
    true = np.max(np.abs(blocks), axis=-1)
    assert np.all(top[big] == 6 * 448 / 64) and np.all(top[big] < true[big])
