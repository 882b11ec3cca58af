"""Pins for the oracle's routing, permutation, grouped GEMM and whole FFN (CPU only)."""

import itertools
import math

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x


# ----------------------------------------------------------------------------- routing

def test_topk_matches_bruteforce_subsets_on_tiny():
    cfg = CONFIGS["tiny"]
    lg = gen_logits(cfg).numpy()
    ids, w = R.route_topk(lg, cfg.k)
    for t in range(cfg.T):
        l64 = lg[t].astype(np.float64)
        p = np.exp(l64 - l64.max())
        p /= p.sum()
        best = max(itertools.combinations(range(cfg.E), cfg.k), key=lambda s: sum(p[list(s)]))
        assert set(ids[t].tolist()) == set(best)
        assert abs(w[t].sum() - 1.0) < 1e-12
        assert np.allclose(w[t], p[ids[t]] / p[ids[t]].sum(), rtol=1e-14)


def test_topk_ties_go_to_lower_id_and_no_renorm():
    lg = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]], dtype=np.float32)
    ids, w = R.route_topk(lg, 2, renormalize=False)
    assert ids.tolist() == [[1, 2]]
    l64 = lg[0].astype(np.float64)
    p = np.exp(l64 - 3.0) / np.exp(l64 - 3.0).sum()
    assert np.allclose(w[0], p[[1, 2]], rtol=1e-12)
    assert abs(w[0, 0] - 1.0 / (3.0 + math.exp(-2.0) + math.exp(-3.0))) < 1e-15


def test_masked_experts_are_never_chosen_and_all_masked_drops():
    lg = np.array([[-np.inf, 0.5, -np.inf, 0.1], [-np.inf] * 4, [0.0, -np.inf, -np.inf, -np.inf]],
                  dtype=np.float32)
    ids, w = R.route_topk(lg, 2)
    assert ids[0].tolist() == [1, 3]
    assert ids[1].tolist() == [-1, -1] and np.all(w[1] == 0)
    assert ids[2].tolist() == [0, -1] and w[2].tolist() == [1.0, 0.0]


def test_permute_offsets_order_and_padding():
    ids = np.array([[2, 0], [0, 2], [2, -1], [1, 2]])
    w = np.arange(8, dtype=np.float64).reshape(4, 2) / 10
    p = R.permute(ids, w, E=4)
    assert p["counts"].tolist() == [2, 1, 4, 0]
    assert p["offs"].tolist() == [0, 128, 256, 384, 384]
    # expert 2 rows: (t0,j0), (t1,j1), (t2,j0), (t3,j1) in that order
    assert p["dst_row"].tolist() == [[256, 0], [1, 257], [258, -1], [128, 259]]
    assert p["row_token"][256:260].tolist() == [0, 1, 2, 3]
    assert p["row_slot"][256:260].tolist() == [0, 3, 4, 7]
    assert p["row_slot"][128] == 6 and np.all(p["row_slot"][2:128] == -1)
    assert np.allclose(p["row_w"][256:260], [0.0, 0.3, 0.4, 0.7])
    assert np.all(p["row_token"][2:128] == -1) and np.all(p["row_w"][2:128] == 0)
    assert p["R"] == 384


# ------------------------------------------------------------------------- grouped GEMM

def test_grouped_gemm_vs_triple_loop():
    rng = np.random.default_rng(7)
    E, N, K = 3, 5, 32
    offs = np.array([0, 128, 128, 256])
    valid = [3, 0, 2]
    a = rng.standard_normal((256, K))
    b = rng.standard_normal((E, N, K))
    c = M.grouped_gemm(a, lambda e: b[e], offs, rows_valid=valid)
    for e in range(E):
        for r in range(offs[e], offs[e] + valid[e]):
            for n in range(N):
                s = 0.0
                for kk in range(K):
                    s += a[r, kk] * b[e, n, kk]
                assert abs(c[r, n] - s) < 1e-12
    assert np.all(c[3:128] == 0)


def _unit_weights(E, N, K, code):
    codes = np.full((E, N, K), code, dtype=np.uint8)
    packed = F.pack_nibbles(codes)
    sf = np.full((E, N, K // 16), 0x38, dtype=np.uint8)  # scale 1.0
    return M.QuantWeights(packed, sf, np.ones(E, np.float32))


def test_grouped_gemm_closed_form_all_ones():
    K, N = 64, 8
    w = _unit_weights(2, N, K, code=2)  # every element 1.0
    a = Q.dequantize(np.full((128, K), 2, np.uint8), np.full((128, K // 16), 0x38, np.uint8), 1.0)
    c = M.grouped_gemm(a, w.dequant, np.array([0, 128, 128]))
    assert np.all(c == K)


def test_grouped_gemm_one_hot_selects_weight_column():
    rng = np.random.default_rng(8)
    K, N = 64, 16
    wf = rng.standard_normal((1, N, K)).astype(np.float32)
    w = M.QuantWeights.from_float(wf)
    a = np.zeros((128, K))
    a[5, 17] = 1.0
    c = M.grouped_gemm(a, w.dequant, np.array([0, 128]))
    assert np.array_equal(c[5], w.dequant(0)[:, 17])


def test_silu_closed_forms():
    assert M.silu_scalar(0.0) == 0.0
    assert abs(M.silu_scalar(1.0) - 1.0 / (1.0 + math.e ** -1)) < 1e-16
    assert M.silu(np.array([-800.0]))[0] == 0.0
    assert M.silu(np.array([50.0]))[0] == pytest.approx(50.0, rel=1e-15)


# ----------------------------------------------------------------------- FFN invariants

def _tiny_inputs(E=8, T=64, H=256, I=128, k=2, seed=0):
    cfg = CONFIGS["tiny"]
    x = gen_x(cfg).float().numpy()[:T, :H]
    lg = gen_logits(cfg).numpy()[:T, :E]
    w1 = M.QuantWeights.from_float(np.stack([gen_weight_expert(seed, 1, e, 2 * I, H).float().numpy() for e in range(E)]))
    w2 = M.QuantWeights.from_float(np.stack([gen_weight_expert(seed, 2, e, H, I).float().numpy() for e in range(E)]))
    return x, lg, w1, w2


@pytest.fixture(scope="module")
def tiny():
    return _tiny_inputs()


def test_dropped_tokens_are_zero(tiny):
    x, lg, w1, w2 = tiny
    ids, w = R.route_topk(lg, 2)
    ids[3] = -1
    ids[10] = -1
    res = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=ids, weights=w)
    assert np.all(res["out"][3] == 0) and np.all(res["out"][10] == 0)
    assert np.all(np.abs(res["out"][4]) > 0)


def test_empty_expert_leaves_no_trace(tiny):
    x, lg, w1, w2 = tiny
    lg2 = lg.copy()
    lg2[:, 5] = -np.inf  # expert 5 gets no token
    r1 = M.moe_ffn(x, lg2, 2, w1, w2, np.float32(64.0))
    assert r1["perm"]["counts"][5] == 0
    # replace expert 5's weights by something else: nothing changes
    w1b = M.QuantWeights(w1.codes.copy(), w1.sf.copy(), w1.gs.copy())
    w1b.codes[5] ^= 0x77
    r2 = M.moe_ffn(x, lg2, 2, w1b, w2, np.float32(64.0))
    assert np.array_equal(r1["out"], r2["out"])


def test_expert_relabeling_invariance(tiny):
    x, lg, w1, w2 = tiny
    perm = np.array([3, 7, 0, 5, 1, 6, 2, 4])  # new id of old expert e is perm[e]
    inv = np.argsort(perm)
    lgp = lg[:, inv]  # column perm[e] of the new logits = old column e
    w1p = M.QuantWeights(w1.codes[inv], w1.sf[inv], w1.gs[inv])
    w2p = M.QuantWeights(w2.codes[inv], w2.sf[inv], w2.gs[inv])
    a = M.moe_ffn(x, lg, 2, w1, w2, np.float32(64.0))["out"]
    b = M.moe_ffn(x, lgp, 2, w1p, w2p, np.float32(64.0))["out"]
    assert np.allclose(a, b, rtol=1e-12, atol=1e-15)


def test_top1_weight1_is_plain_expert_ffn(tiny):
    x, lg, w1, w2 = tiny
    gs_h = np.float32(64.0)
    ids = np.argmax(lg, axis=1)[:, None].astype(np.int32)
    w = np.ones((x.shape[0], 1))
    res = M.moe_ffn(x, None, 1, w1, w2, gs_h, ids=ids, weights=w)
    gs_x = Q.global_scale(x)
    xc, xsf = Q.quantize(x, gs_x)
    xd = Q.dequantize(xc, xsf, gs_x)
    for t in range(0, x.shape[0], 7):
        e = ids[t, 0]
        c1 = xd[t] @ w1.dequant(e).T
        I = c1.shape[0] // 2
        h = (c1[:I] / (1 + np.exp(-c1[:I])) * c1[I:]).astype(np.float32)[None]
        hc, hsf = Q.quantize(h, gs_h)
        y = Q.dequantize(hc, hsf, gs_h)[0] @ w2.dequant(e).T
        assert np.allclose(res["out"][t], y, rtol=1e-13, atol=1e-14)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(9)
    v = rng.standard_normal(10000) * 100
    v = np.concatenate([v, [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]])
    t = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(M.bf16_round(v), t)


# ------------------------------------------------- routing weight and the FFN composition
#
# The pages scatter each expert's output back to its token with the routing weight
# ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our Adaptation": scatter with routing
# weights; section "Phase 3: Full MoE pipeline") after L1 -> SwiGLU -> FP4 -> L2.  These pins
# fix that composition without restating moe_ffn's formula: a worked example whose every
# intermediate is derived by hand below from the format definitions, and two relations the
# weighted sum must obey whatever the experts compute.

E2M1_CODE = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def _codes_of(values):
    """E2M1 codes (sign in bit 3) of values already on the E2M1 grid."""
    return np.array([E2M1_CODE[abs(v)] | (8 if v < 0 else 0) for v in values], dtype=np.uint8)


def _unit_scale_weights(mats):
    """QuantWeights from float matrices on the E2M1 grid: block scales 1.0 (E4M3 0x38) and
    global scales 1, so each dequantized element is exactly the given value."""
    mats = np.asarray(mats, dtype=np.float64)
    E, N, K = mats.shape
    codes = np.stack([_codes_of(m.ravel()).reshape(N, K) for m in mats])
    return M.QuantWeights(F.pack_nibbles(codes), np.full((E, N, K // 16), 0x38, np.uint8),
                          np.ones(E, np.float32))


# W2 column 0 of the two experts (every other W2 entry is 0)
C0 = [1.0, -2.0, 0.5, 3.0, 0.0, -6.0, 4.0, 1.5, -1.0, 2.0, -0.5, -3.0, 6.0, 0.0, -4.0, 1.0]
C1 = [-1.0, 0.5, 2.0, -3.0, 6.0, 1.0, -0.5, 0.0, 4.0, -2.0, 1.5, 3.0, -6.0, 1.0, 0.5, -4.0]


def _worked_example():
    """One token, H = I = 16, two experts, both chosen with weights (0.25, 0.75).

    x = (6, 0, ..., 0): gs_x = 2688 / 6 = 448; the block scale (6/6)*448 = 448 is E4M3's largest
    value, d = 448, so x*gs_x/d = x and the codes hold x exactly: x dequantizes to itself.
    W1 of expert e has gate row 0 = (a_e, 0, ...), up row 0 = (b_e, 0, ...), all else 0, so
    gate_0 = 6*a_e, up_0 = 6*b_e and every other h feature is silu(0)*up = 0.
      expert 0: a = 1,   b = 0.5 -> g = 6, u = 3  -> h_0 = 18 / (1 + e^-6) = 17.9555
      expert 1: a = 0.5, b = 2   -> g = 3, u = 12 -> h_0 = 36 / (1 + e^-3) = 34.2927
    Re-quantized with gs_h = 1 (a single nonzero element in the block):
      expert 0: s = 17.9555/6 = 2.9926 -> nearest E4M3 is 3.0 (byte 0x44); h_0/3 = 5.985 rounds
                to E2M1 6, so h_0 dequantizes to 6 * 3 = 18
      expert 1: s = 34.2927/6 = 5.7154 -> below the 5.75 midpoint of 5.5 and 6.0, so 5.5 (0x4B);
                h_0/5.5 = 6.235 saturates to 6, so h_0 dequantizes to 6 * 5.5 = 33
    W2 of expert e has column 0 = C_e, all else 0, so Y_e = hq_0 * C_e, and
      out = 0.25 * 18 * C0 + 0.75 * 33 * C1 = 4.5 * C0 + 24.75 * C1   (exact in float64)."""
    H = I = 16
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 6.0
    w1 = np.zeros((2, 2 * I, H))
    w1[0, 0, 0], w1[0, I, 0] = 1.0, 0.5
    w1[1, 0, 0], w1[1, I, 0] = 0.5, 2.0
    w2 = np.zeros((2, H, I))
    w2[0, :, 0], w2[1, :, 0] = C0, C1
    ids = np.array([[0, 1]], np.int32)
    weights = np.array([[0.25, 0.75]])
    return x, _unit_scale_weights(w1), _unit_scale_weights(w2), ids, weights


def test_worked_example_by_hand():
    x, w1, w2, ids, weights = _worked_example()
    res = M.moe_ffn(x, None, 2, w1, w2, np.float32(1.0), ids=ids, weights=weights, keep=True)
    assert res["gs_x"] == np.float32(448.0)
    expected = 4.5 * np.array(C0) + 24.75 * np.array(C1)
    assert np.array_equal(res["out"][0], expected)
    # the intermediates derived above: expert 0's row is 0, expert 1's row is 128
    assert res["h_sf"][0, 0] == 0x44 and res["h_sf"][128, 0] == 0x4B
    assert res["h_codes"][0, 0] == 7 and res["h_codes"][128, 0] == 7
    assert np.all(res["h_codes"][[0, 128], 1:] == 0)


def test_both_slots_on_one_expert_equal_its_single_slot_ffn(tiny):
    """Weights 0.25 and 0.75 on the same expert add up to that expert's output once (weight 1),
    not twice, whatever the expert computes."""
    x, lg, w1, w2 = tiny
    T = x.shape[0]
    e = np.argmax(lg, axis=1).astype(np.int32)
    two = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=np.stack([e, e], 1),
                    weights=np.tile([0.25, 0.75], (T, 1)))["out"]
    one = M.moe_ffn(x, None, 1, w1, w2, np.float32(64.0), ids=e[:, None],
                    weights=np.ones((T, 1)))["out"]
    assert np.abs(one).max() > 0
    assert np.allclose(two, one, rtol=1e-14, atol=1e-15 * np.abs(one).max())


def test_output_is_linear_in_the_routing_weights(tiny):
    """Scaling every routing weight by 2 scales the output by exactly 2 (a power of two is exact
    in float64); by 3, to within float64 rounding.  The experts' outputs do not depend on the
    weights, so only a weight applied once, linearly, passes."""
    x, lg, w1, w2 = tiny
    ids, w = R.route_topk(lg, 2)
    base = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=ids, weights=w)["out"]
    twice = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=ids, weights=2 * w)["out"]
    thrice = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=ids, weights=3 * w)["out"]
    assert np.abs(base).max() > 0
    assert np.array_equal(twice, 2 * base)
    assert np.allclose(thrice, 3 * base, rtol=1e-14, atol=1e-15 * np.abs(base).max())
    # and a weight of 0 on one slot leaves exactly the other slot's weighted output
    w0 = w.copy()
    w0[:, 1] = 0.0
    only0 = M.moe_ffn(x, None, 2, w1, w2, np.float32(64.0), ids=ids, weights=w0)["out"]
    ids_1 = ids[:, :1]
    alone = M.moe_ffn(x, None, 1, w1, w2, np.float32(64.0), ids=ids_1, weights=w[:, :1])["out"]
    # (the two calls bucket different row counts per expert, so BLAS may sum in another order)
    assert np.allclose(only0, alone, rtol=1e-14, atol=1e-15 * np.abs(alone).max())
