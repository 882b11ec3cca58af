"""Pins for the oracle's MXFP4 quantizer (CPU only): UE8M0 decode against the library type,
the scale exponent's defining inequality and closed forms, the round trip on grid blocks,
saturation, and the per-element error bound."""

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import mx as X
from oracle import quant as Q


def test_e8m0_decode_matches_the_library_type():
    b = torch.arange(256, dtype=torch.uint8)
    t = b.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ours = X.e8m0_decode(np.arange(256))
    assert np.isnan(ours[255]) and np.isnan(t[255])
    assert np.array_equal(ours[:255], t[:255])
    assert ours[127] == 1.0 and ours[0] == 2.0 ** -127 and ours[254] == 2.0 ** 127


def test_block_exponent_closed_forms():
    cases = {6.0: 0, 4.0: 0, 7.99: 0, 8.0: 1, 3.99: -1, 1.0: -2, 0.5: -3, 448.0: 6,
             0.0: -127, 2.0 ** -200: -127, 2.0 ** 200: 127}
    for a, e in cases.items():
        assert int(X.block_exponent(a)) == e, a


def test_block_exponent_defining_inequality():
    """2^(e+2) <= amax < 2^(e+3): the block's largest element lands in [4, 8) after scaling."""
    rng = np.random.default_rng(0)
    a = np.exp(rng.uniform(-60, 60, 5000))
    e = X.block_exponent(a)
    assert np.all(np.ldexp(1.0, e + 2) <= a) and np.all(a < np.ldexp(1.0, e + 3))


@pytest.mark.parametrize("e", [-20, -3, 0, 5, 40])
def test_round_trip_on_grid_blocks(e):
    """Blocks on the E2M1 grid times 2^e come back exactly; when the block's largest magnitude is
    4 or 6 the scale byte is e + 127."""
    rng = np.random.default_rng(e + 100)
    codes = rng.integers(0, 16, size=(6, 64)).astype(np.uint8)
    codes[:, ::32] = rng.choice(np.array([6, 7, 14, 15], np.uint8), size=(6, 2))  # +-4 or +-6
    x = np.ldexp(F.e2m1_decode(codes), e)
    c2, s2 = X.quantize_mxfp4(x)
    assert np.all(s2 == e + 127)
    assert np.array_equal(X.dequantize_mxfp4(c2, s2), x)
    # a block whose largest magnitude is 3 gets half the scale and the same values
    small = np.ldexp(np.array([[3.0, -1.5, 0.5, 2.0] * 8]), e)
    c3, s3 = X.quantize_mxfp4(small)
    assert s3[0, 0] == e + 126 and np.array_equal(X.dequantize_mxfp4(c3, s3), small)


def test_saturation_clips_to_six_times_the_scale():
    x = np.zeros((1, 32))
    x[0, 0] = 7.5
    x[0, 1] = -7.0
    x[0, 2] = 5.0
    c, s = X.quantize_mxfp4(x)
    assert s[0, 0] == 127  # amax 7.5 in [4, 8): e = 0
    d = X.dequantize_mxfp4(c, s)
    assert d[0, 0] == 6.0 and d[0, 1] == -6.0 and d[0, 2] == 4.0  # 5 ties to the even code (4)


def test_error_bound_per_element():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 256)) * 3.0
    c, s = X.quantize_mxfp4(x)
    d = X.dequantize_mxfp4(c, s)
    scale = np.repeat(X.e8m0_decode(s), 32, axis=1)
    y = np.abs(x) / scale
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    bound = np.where(y <= 6, half_step, y - 6) * scale
    assert np.all(np.abs(x - d) <= bound * (1 + 1e-12))


def test_nvfp4_is_finer_than_mxfp4_on_gaussian_data():
    """The pages pick NVFP4 over MXFP4; with 16-element E4M3-scaled blocks its error on N(0,1)
    data is lower than with 32-element power-of-two blocks."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    gs = Q.global_scale(x)
    nv = Q.dequantize(*Q.quantize(x, gs), gs)
    mx = X.dequantize_mxfp4(*X.quantize_mxfp4(x))
    err = lambda d: np.linalg.norm(d - x) / np.linalg.norm(x)  # noqa: E731
    assert err(nv) < err(mx)
