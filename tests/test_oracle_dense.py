"""Pins for the oracle's RMSNorm, fused RMSNorm + quantize and dense NVFP4 linear (CPU only)."""

import itertools

import numpy as np
import pytest
import torch

from oracle import dense as D
from oracle import formats as F
from oracle import quant as Q


def _bf16_values(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("eps", [0.0, 1e-6, 1e-2])
def test_rmsnorm_matches_the_library_routine_in_float64(eps):
    """torch's rms_norm evaluated in float64 is the textbook value; the oracle's float32 result
    lies within a few float32 roundings of it."""
    x = _bf16_values((37, 192), seed=1, scale=3.0)
    gamma = _bf16_values((192,), seed=2) + np.float32(1.0)
    y, rstd = D.rmsnorm(x, gamma, eps)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (192,),
                                       weight=torch.from_numpy(gamma).double(), eps=eps).numpy()
    assert y.dtype == np.float32 and rstd.shape == (37,)
    assert np.all(np.abs(y - ref) <= 4 * np.finfo(np.float32).eps * np.abs(ref) + 1e-30)
    exact_rstd = 1.0 / np.sqrt(np.mean(x.astype(np.float64) ** 2, axis=1) + eps)
    assert np.allclose(rstd, exact_rstd, rtol=3e-7, atol=0)


def test_rmsnorm_closed_forms():
    # a constant row of a power of two: mean(x^2) = c^2 exactly, so y = sign(c) * gamma
    x = np.full((2, 64), 0.25, dtype=np.float32)
    x[1] = -8.0
    gamma = np.linspace(-2, 2, 64).astype(np.float32)
    y, rstd = D.rmsnorm(x, gamma, 0.0)
    assert np.array_equal(rstd, np.array([4.0, 0.125], np.float32))
    assert np.array_equal(y[0], gamma) and np.array_equal(y[1], -gamma)
    # eps enters under the root: x = 1 everywhere, eps = 3 -> rstd = 1 / sqrt(4) = 0.5
    y, rstd = D.rmsnorm(np.ones((1, 32), np.float32), np.full(32, 3.0, np.float32), 3.0)
    assert rstd[0] == 0.5 and np.all(y == 1.5)
    # a single nonzero element: mean = v^2 / cols
    x = np.zeros((1, 64), np.float32)
    x[0, 5] = 2.0
    y, rstd = D.rmsnorm(x, np.ones(64, np.float32), 0.0)
    assert rstd[0] == np.float32(1.0 / np.sqrt(4.0 / 64))  # = 1 / 0.25 = 4
    assert y[0, 5] == 8.0 and np.count_nonzero(y) == 1
    # an all-zero row with eps = 0 gives 1/0 = inf and 0 * inf = NaN (no hidden clamp)
    y, rstd = D.rmsnorm(np.zeros((1, 16), np.float32), np.ones(16, np.float32), 0.0)
    assert np.isinf(rstd[0]) and np.all(np.isnan(y))


@pytest.mark.parametrize("n", [-6, -1, 3, 9])
def test_rmsnorm_is_exactly_invariant_to_power_of_two_scaling(n):
    """With eps = 0 every step scales by an exact power of two, so x * 2^n normalizes to the
    same bits as x (a stray cols factor, an eps in the wrong place or a missing root breaks it)."""
    x = _bf16_values((9, 128), seed=7)
    gamma = _bf16_values((128,), seed=8)
    y0, r0 = D.rmsnorm(x, gamma, 0.0)
    y1, r1 = D.rmsnorm(x * np.float32(2.0 ** n), gamma, 0.0)
    assert np.array_equal(y0, y1)
    assert np.array_equal(r1, r0 * np.float32(2.0 ** -n))


def test_rmsnorm_quantize_takes_gs_from_the_normalized_tensor():
    x = _bf16_values((16, 256), seed=4, scale=5.0)
    gamma = _bf16_values((256,), seed=5, scale=0.5)
    codes, sf, gs, y = D.rmsnorm_quantize(x, gamma, 1e-6)
    assert gs == Q.global_scale(y) and gs != Q.global_scale(x)
    # the block holding max|y| gets the largest E4M3 scale (448 = 0x7E), by the choice of gs
    r, c = np.unravel_index(np.argmax(np.abs(y)), y.shape)
    assert sf[r, c // 16] == 0x7E
    c2, sf2 = Q.quantize(y, gs)
    assert np.array_equal(codes, c2) and np.array_equal(sf, sf2)


def _grid_activation(rng, M, K):
    """Activations exactly on the NVFP4 grid with gs = 1: every block is E2M1 codes times an
    E4M3 scale d with one element at +-6 d (so the block scale comes back as d), and block 0
    has d = 448, whose +6 element 2688 makes amax give gs = 2688 / 2688 = 1."""
    codes = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    codes[:, ::16] = rng.choice(np.array([7, 15], np.uint8), size=(M, K // 16))
    codes[0, 0] = 7
    sfb = rng.choice(np.array([0x30, 0x38, 0x3C, 0x41, 0x4A], np.uint8), size=(M, K // 16))
    sfb[0, 0] = 0x7E
    d = F.e4m3_decode(sfb)
    x = F.e2m1_decode(codes).reshape(M, K // 16, 16) * d[..., None]
    x = x.reshape(M, K)
    assert x[0, 0] == 6.0 * 448.0 and np.max(np.abs(x)) == 2688.0
    return x.astype(np.float32)


def test_linear_equals_a_triple_loop_on_grid_inputs():
    """Grid-exact activations quantize without error, so the linear is the plain product with
    the dequantized weight; a non-square (M, N, K) catches a transposed operand."""
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 32
    x = _grid_activation(rng, M, K)
    w_codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    w_sf = rng.choice(np.array([0x28, 0x30, 0x38, 0x40], np.uint8), size=(N, K // 16))
    gs_w = np.float32(4.0)
    out, aq = D.linear(x, w_codes, w_sf, gs_w)
    assert aq["gs"] == 1.0
    assert np.array_equal(Q.dequantize(aq["codes"], aq["sf"], aq["gs"]), x.astype(np.float64))
    w = F.e2m1_decode(w_codes).reshape(N, K // 16, 16) * F.e4m3_decode(w_sf)[..., None] / 4.0
    w = w.reshape(N, K)
    want = np.zeros((M, N))
    for m, n in itertools.product(range(M), range(N)):
        acc = 0.0
        for kk in range(K):
            acc += float(x[m, kk]) * float(w[n, kk])
        want[m, n] = acc
    assert np.array_equal(out, want)  # small integers and dyadic scales: every sum is exact


def test_linear_one_hot_row_selects_a_weight_column():
    rng = np.random.default_rng(12)
    K, N = 64, 8
    # 2688 = 6 * 448 sets gs = 1; -1344 = -6 * 224 quantizes exactly with block scale 224
    x = np.zeros((2, K), np.float32)
    x[0, 17] = 2688.0
    x[1, 40] = -1344.0
    w_codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    w_sf = np.full((N, K // 16), 0x38, np.uint8)
    out, _ = D.linear(x, w_codes, w_sf, np.float32(1.0))
    w = F.e2m1_decode(w_codes)
    assert np.array_equal(out[0], 2688.0 * w[:, 17])
    assert np.array_equal(out[1], -1344.0 * w[:, 40])


def test_shared_expert_is_the_per_row_ffn():
    """The shared expert evaluated row by row from the definitions: normalize, quantize with the
    batch's global scale, L1, SwiGLU, re-quantize with gs_h, L2 (weight 1, no routing)."""
    from oracle import moe as M
    H, I, Mr = 128, 64, 9
    x = _bf16_values((Mr, H), seed=21)
    gamma = _bf16_values((H,), seed=22) + np.float32(1.0)
    w1 = M.QuantWeights.from_float(_bf16_values((1, 2 * I, H), seed=23, scale=0.05))
    w2 = M.QuantWeights.from_float(_bf16_values((1, H, I), seed=24, scale=0.05))
    gs_h = np.float32(16.0)
    out = D.shared_expert(x, w1, w2, gs_h, gamma=gamma, eps=1e-6)
    y, _ = D.rmsnorm(x, gamma, 1e-6)
    gs_x = Q.global_scale(y)
    xd = Q.dequantize(*Q.quantize(y, gs_x), gs_x)
    for t in range(Mr):
        c1 = xd[t] @ w1.dequant(0).T
        h = (c1[:I] / (1 + np.exp(-c1[:I])) * c1[I:]).astype(np.float32)[None]
        hd = Q.dequantize(*Q.quantize(h, gs_h), gs_h)[0]
        assert np.allclose(out[t], hd @ w2.dequant(0).T, rtol=1e-13, atol=1e-14)
    # without gamma the input is used as given
    plain = D.shared_expert(x, w1, w2, gs_h)
    assert not np.allclose(plain, out)
