"""Pins for the oracle's E2M1 / E4M3 codecs (CPU only).

Each check is independent of the code it tests: the page's printed E2M1 table, brute-force
nearest-value search over the whole code space, and torch's own float8_e4m3fn cast.
"""

import itertools
import os

import numpy as np
import pytest
import torch

from oracle import formats as F


def _load_e2m1_golden(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "e2m1_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((int(c), float(v)))
    return rows


def test_e2m1_decode_matches_page_table(golden_dir):
    rows = _load_e2m1_golden(golden_dir)
    assert len(rows) == 16
    codes = np.array([c for c, _ in rows], dtype=np.uint8)
    want = np.array([v for _, v in rows])
    got = F.e2m1_decode(codes)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))  # -0 for code 8


def test_e2m1_value_set_is_the_pages():
    mags = sorted(set(np.abs(F.e2m1_decode(np.arange(16, dtype=np.uint8))).tolist()))
    assert mags == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


@pytest.mark.parametrize("y,code", [
    (0.0, 0), (-0.0, 8), (0.25, 0), (0.2499, 0), (0.2501, 1), (0.75, 2), (1.25, 2), (1.75, 4),
    (2.5, 4), (3.5, 6), (5.0, 6), (5.0001, 7), (6.0, 7), (7.0, 7), (1e30, 7), (np.inf, 7),
    (-0.25, 8), (-0.75, 10), (-5.0, 14), (-100.0, 15), (-np.inf, 15), (-1e-30, 8),
])
def test_e2m1_encode_ties_and_saturation(y, code):
    assert int(F.e2m1_encode(np.float32(y))) == code


def test_e2m1_encode_idempotent_on_grid():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(codes)), codes)


def _nearest_even(vals, codes, y, is_even):
    """Brute force: nearest representable value, ties to the code with the even mantissa."""
    out = np.empty(len(y), dtype=np.int64)
    for i, v in enumerate(y):
        dist = np.abs(vals - v)
        best = np.min(dist)
        cand = [c for c, d in zip(codes, dist) if d == best]
        if len(cand) > 1:
            cand = [c for c in cand if is_even(c)]
        assert len(cand) == 1, (v, cand)
        out[i] = cand[0]
    return out


def test_e2m1_encode_bruteforce():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.uniform(0, 6, 4000), np.arange(0, 6.01, 0.125), rng.uniform(0, 1, 500)])
    y = y.astype(np.float32).astype(np.float64)
    codes = np.arange(8)
    vals = F.e2m1_decode(codes.astype(np.uint8))
    want = _nearest_even(vals, codes, y, lambda c: c % 2 == 0)
    assert np.array_equal(F.e2m1_encode(y), want)
    assert np.array_equal(F.e2m1_encode(-y), np.where(True, want | 8, 0))


def test_nibble_packing_order():
    c = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    p = F.pack_nibbles(c)
    assert p.tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_nibbles(p), c)


def test_e4m3_decode_code_space():
    v = F.e4m3_decode(np.arange(256, dtype=np.uint8))
    nan = np.isnan(v)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    fin = v[~nan]
    assert np.max(fin) == 448.0 and np.min(fin) == -448.0
    assert v[1] == 2.0 ** -9 and v[0x08] == 2.0 ** -6 and v[0x38] == 1.0
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)  # positive codes are monotone
    assert np.array_equal(v[0x80:0xFF], -v[:0x7F])


def test_e4m3_decode_matches_torch():
    b = torch.arange(256, dtype=torch.uint8)
    t = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(t), np.isnan(ours))
    ok = ~np.isnan(t)
    assert np.array_equal(t[ok], ours[ok])


def test_e4m3_encode_matches_torch_cast():
    pos = F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(1)
    v = np.concatenate([pos, mids, rng.uniform(0, 448, 20000), np.exp(rng.uniform(-12, 6, 20000))])
    v = v[v <= 448].astype(np.float32)
    v = np.concatenate([v, -v])
    t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(v), t)


def test_e4m3_encode_bruteforce_and_saturation():
    codes = np.arange(0x7F)
    vals = F.e4m3_decode(codes.astype(np.uint8))
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-12, 6, 3000))])
    v = v[v < 448].astype(np.float32).astype(np.float64)
    want = _nearest_even(vals, codes, v, lambda c: c % 2 == 0)
    assert np.array_equal(F.e4m3_encode(v), want)
    for big in (448.0, 449.0, 470.0, 1e9, np.inf):
        assert int(F.e4m3_encode(np.float32(big))) == 0x7E
    assert int(F.e4m3_encode(np.float32(np.nan))) == 0x7F
    assert int(F.e4m3_encode(np.float32(2.0 ** -10))) == 0      # tie between 0 and 2^-9 -> 0
    assert int(F.e4m3_encode(np.float32(3 * 2.0 ** -10))) == 2  # tie between 2^-9 and 2^-8 -> 2^-8
    assert int(F.e4m3_encode(np.float32(3 * 2.0 ** -11))) == 1  # 0.75 * 2^-9 -> nearest 2^-9


def test_every_pair_of_adjacent_e2m1_values_has_its_midpoint_tested():
    vals = F.e2m1_decode(np.arange(8, dtype=np.uint8))
    for a, b in itertools.pairwise(vals):
        mid = np.float32((a + b) / 2)
        c = int(F.e2m1_encode(mid))
        ca, cb = int(F.e2m1_encode(a)), int(F.e2m1_encode(b))
        assert c in (ca, cb) and c % 2 == 0
