"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in the oracle (a wrong formula put in place of an oracle function
for the duration of the test) and runs the pins that guard that function: at least one of them
has to fail.  This checks the pins, not the oracle; the oracle itself is never edited.
"""

import numpy as np
import pytest

from oracle import dense as D
from oracle import formats as F
from oracle import moe as M
from oracle import mx as MX
from oracle import quant as Q
from oracle import routing as R
from tests import test_oracle_dense as PD
from tests import test_oracle_formats as PF
from tests import test_oracle_mx as PMX
from tests import test_oracle_quant as PQ
from tests import test_oracle_routing_moe as PR


def _rmsnorm_mutant(kind):
    """RMSNorm with one planted mistake: the sum of squares instead of their mean, eps outside
    the root, or gamma left out."""
    def f(x, gamma, eps):
        x32 = np.asarray(x, dtype=np.float32)
        g32 = np.asarray(gamma, dtype=np.float32)
        x64 = x32.astype(np.float64)
        ss = np.sum(x64 * x64, axis=1)
        ms = (ss if kind == "sum" else ss / x32.shape[1]).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
            if kind == "eps_outside":
                rstd = (np.float32(1.0) / (np.sqrt(ms).astype(np.float32) + np.float32(eps)))
            else:
                rstd = np.float32(1.0) / np.sqrt((ms + np.float32(eps)).astype(np.float32))
            rstd = rstd.astype(np.float32)
            y = (x32 * rstd[:, None]).astype(np.float32)
            if kind != "no_gamma":
                y = (y * g32[None, :]).astype(np.float32)
        return y, rstd
    return f


def _linear_weight_scale_ignored(x, w_codes, w_sf, gs_w):
    return D.__dict__["_orig_linear"](x, w_codes, w_sf, np.float32(1.0))


def _global_scale_wrong_numerator(x):
    a = np.max(np.abs(np.asarray(x, dtype=np.float32))) if np.size(x) else np.float32(0)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        gs = np.float32(np.float32(448.0) / np.float32(a))
    return gs if np.isfinite(gs) and gs > 0 else np.float32(1.0)


def _scale_from_amax_wrong_numerator(amax):
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        gs = np.float32(np.float32(448.0) / np.float32(amax))
    return gs if np.isfinite(gs) and gs > 0 else np.float32(1.0)


def _clipping_at_or_above_448(x, gs):
    """Counts a block scale of exactly 448 as saturated (the boundary on the wrong side)."""
    x32 = np.asarray(x, dtype=np.float32)
    rows, cols = x32.shape
    a_b = np.max(np.abs(x32.reshape(rows, cols // 16, 16)), axis=-1)
    s = ((a_b / np.float32(6.0)).astype(np.float32) * np.float32(gs)).astype(np.float32)
    under = int(np.count_nonzero((a_b > 0) & (F.e4m3_encode(s) & 0x7F == 0)))
    return int(np.count_nonzero(s >= np.float32(448.0))), under


def _route_without_renormalization(logits, k, renormalize=True):
    return R.__dict__["_orig_route_topk"](logits, k, renormalize=False)


def _permute_descending_tokens(ids, w, E):
    ids = np.asarray(ids)
    T = ids.shape[0]
    p = R.__dict__["_orig_permute"](ids[::-1], np.asarray(w)[::-1], E)
    p["dst_row"] = p["dst_row"][::-1]
    p["row_token"] = np.where(p["row_token"] >= 0, T - 1 - p["row_token"], -1)
    return p


def _silu_is_sigmoid(g):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-np.asarray(g, dtype=np.float64)))


def _e2m1_ties_away_from_zero(y):
    """E2M1 encoder rounding halfway cases away from zero instead of to the even code."""
    y = np.asarray(y, dtype=np.float64)
    vals = F.e2m1_decode(np.arange(8, dtype=np.uint8))
    a = np.minimum(np.abs(y), 6.0)
    idx = np.searchsorted(vals, a, side="left")
    idx = np.clip(idx, 0, 7)
    lo = np.clip(idx - 1, 0, 7)
    pick = np.where(np.abs(vals[lo] - a) < np.abs(vals[idx] - a), lo, idx)
    sign = np.where(np.signbit(y), 8, 0)
    return (pick | sign).astype(np.uint8)


def _e4m3_no_saturation(v):
    """E4M3 encoder that returns the NaN code past 448 instead of saturating."""
    out = F.__dict__["_orig_e4m3_encode"](v)
    big = np.abs(np.asarray(v, dtype=np.float64)) > 448
    return np.where(big, np.uint8(0x7F), out).astype(np.uint8)


def _sf_offset_rows_not_interleaved(r, c, n_sf_cols):
    """Tile map with rows 0..127 of an atom laid out in order (r % 128) * 4 + c % 4."""
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    atom = (r // 128) * (n_sf_cols // 4) + (c // 4)
    return atom * 512 + (r % 128) * 4 + (c % 4)


def _grouped_gemm_wrong_expert(a, b_dequant, offs, rows_valid=None):
    """Grouped GEMM that multiplies every segment by the first expert's weights."""
    return M.__dict__["_orig_grouped_gemm"](a, lambda e: b_dequant(0), offs, rows_valid)


def _ffn_weight_omitted(x, logits, k, w1, w2, gs_h, renormalize=True, ids=None, weights=None,
                        **kw):
    """The expert FFN with the routing weight left out of the scatter (every slot at weight 1)."""
    if ids is None:
        ids, weights = R.route_topk(logits, k, renormalize)
    return M.__dict__["_orig_moe_ffn"](x, None, k, w1, w2, gs_h, ids=ids,
                                       weights=np.ones_like(np.asarray(weights, np.float64)), **kw)


class _GateUpSwapped:
    """W1 whose gate rows [0, I) and up rows [I, 2I) trade places: silu(up) * gate."""

    def __init__(self, w):
        self.w, self.E, self.N = w, w.E, w.N

    def dequant(self, e):
        d = self.w.dequant(e)
        half = d.shape[0] // 2
        return np.concatenate([d[half:], d[:half]])


def _ffn_gate_up_swapped(x, logits, k, w1, w2, gs_h, **kw):
    return M.__dict__["_orig_moe_ffn"](x, logits, k, _GateUpSwapped(w1), w2, gs_h, **kw)


def _ffn_requant_with_gs_x(x, logits, k, w1, w2, gs_h, **kw):
    """The intermediate re-quantized with the activations' global scale in place of gs_h."""
    gs_x = kw.get("gs_x")
    if gs_x is None:
        gs_x = Q.global_scale(np.asarray(x, np.float32))
    return M.__dict__["_orig_moe_ffn"](x, logits, k, w1, w2, np.float32(gs_x), **kw)


def _mx_exponent_rounded_up(amax):
    """ceil(log2(amax)) - 2 in place of floor: the block's largest element lands in (2, 4]."""
    a = np.asarray(amax, dtype=np.float64)
    with np.errstate(divide="ignore"):
        e = np.ceil(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64) - 2
    return np.clip(np.where(a > 0, e, -127), -127, 127)


def _mx_exponent_emax3(amax):
    """floor(log2(amax)) - 3: the exponent of E2M1's largest value taken as 3."""
    return np.clip(MX.__dict__["_orig_block_exponent"](amax) - 1, -127, 127)


def _pins_mx():
    return [PMX.test_block_exponent_closed_forms, PMX.test_block_exponent_defining_inequality,
            lambda: PMX.test_round_trip_on_grid_blocks(5), PMX.test_saturation_clips_to_six_times_the_scale]


def _pins_formats():
    return [PF.test_e2m1_encode_bruteforce,
            lambda: PF.test_e2m1_encode_ties_and_saturation(2.5, 4),
            PF.test_e4m3_encode_bruteforce_and_saturation,
            PF.test_e4m3_encode_matches_torch_cast]


def _pins_tile_map():
    return [PQ.test_sf_tile_offsets_hand_worked, PQ.test_sf_tile_is_bijection_and_inverse]


def _pins_gemm():
    return [PR.test_grouped_gemm_vs_triple_loop, PR.test_grouped_gemm_closed_form_all_ones,
            PR.test_grouped_gemm_one_hot_selects_weight_column]


def _pins_dense_rmsnorm():
    return [lambda: PD.test_rmsnorm_matches_the_library_routine_in_float64(1e-6),
            PD.test_rmsnorm_closed_forms,
            lambda: PD.test_rmsnorm_is_exactly_invariant_to_power_of_two_scaling(3),
            PD.test_rmsnorm_quantize_takes_gs_from_the_normalized_tensor,
            PD.test_shared_expert_is_the_per_row_ffn]


def _pins_dense_linear():
    return [PD.test_linear_equals_a_triple_loop_on_grid_inputs,
            PD.test_linear_one_hot_row_selects_a_weight_column]


def _pins_quant():
    return [PQ.test_global_scale_closed_forms,
            lambda: PQ.test_round_trip_on_grid_blocks(0x38, 1.0),
            PQ.test_round_tripped_scale_differs_from_raw_scale]


def _pins_hscale():
    return [PQ.test_scale_from_amax_closed_forms,
            PQ.test_delayed_scale_from_the_same_data_is_the_dynamic_scale,
            PQ.test_block_scale_clipping_hand_cases,
            PQ.test_block_scale_clipping_agrees_with_the_quantizer]


def _pins_routing():
    return [PR.test_topk_matches_bruteforce_subsets_on_tiny,
            PR.test_topk_ties_go_to_lower_id_and_no_renorm,
            PR.test_permute_offsets_order_and_padding]


def _pins_ffn():
    tiny = PR._tiny_inputs()
    return [PR.test_silu_closed_forms, lambda: PR.test_top1_weight1_is_plain_expert_ffn(tiny),
            PR.test_worked_example_by_hand,
            lambda: PR.test_both_slots_on_one_expert_equal_its_single_slot_ffn(tiny),
            lambda: PR.test_output_is_linear_in_the_routing_weights(tiny)]


MUTANTS = [
    ("rmsnorm: sum of squares, not the mean", D, "rmsnorm", _rmsnorm_mutant("sum"),
     _pins_dense_rmsnorm),
    ("rmsnorm: eps outside the square root", D, "rmsnorm", _rmsnorm_mutant("eps_outside"),
     _pins_dense_rmsnorm),
    ("rmsnorm: gamma left out", D, "rmsnorm", _rmsnorm_mutant("no_gamma"), _pins_dense_rmsnorm),
    ("linear: the weight's global scale ignored", D, "linear", _linear_weight_scale_ignored,
     _pins_dense_linear),
    ("quantizer: 448 / amax as the global scale", Q, "global_scale",
     _global_scale_wrong_numerator, _pins_quant),
    ("quantizer: codes against the raw block scale", Q, "quantize", Q.quantize_raw_scale,
     _pins_quant),
    ("delayed scale: 448 / amax", Q, "scale_from_amax", _scale_from_amax_wrong_numerator,
     _pins_hscale),
    ("clipping count: a scale of exactly 448 counted as saturated", Q, "block_scale_clipping",
     _clipping_at_or_above_448, _pins_hscale),
    ("routing: weights not renormalized over the k", R, "route_topk",
     _route_without_renormalization, _pins_routing),
    ("permutation: tokens in descending order inside an expert", R, "permute",
     _permute_descending_tokens, _pins_routing),
    ("SwiGLU: sigmoid(g) in place of silu(g)", M, "silu", _silu_is_sigmoid, _pins_ffn),
    ("FFN: routing weight left out of the scatter", M, "moe_ffn", _ffn_weight_omitted,
     _pins_ffn),
    ("FFN: gate and up projections swapped", M, "moe_ffn", _ffn_gate_up_swapped, _pins_ffn),
    ("FFN: intermediate re-quantized with gs_x for gs_h", M, "moe_ffn", _ffn_requant_with_gs_x,
     _pins_ffn),
    ("E2M1: halfway cases away from zero", F, "e2m1_encode", _e2m1_ties_away_from_zero,
     _pins_formats),
    ("E4M3: NaN instead of saturation past 448", F, "e4m3_encode", _e4m3_no_saturation,
     _pins_formats),
    ("scale tiles: rows of an atom not interleaved by 32", Q, "sf_tile_offset",
     _sf_offset_rows_not_interleaved, _pins_tile_map),
    ("grouped GEMM: every segment against expert 0", M, "grouped_gemm",
     _grouped_gemm_wrong_expert, _pins_gemm),
    ("MXFP4: the scale exponent rounded up", MX, "block_exponent", _mx_exponent_rounded_up,
     _pins_mx),
    ("MXFP4: 3 as E2M1's largest exponent", MX, "block_exponent", _mx_exponent_emax3, _pins_mx),
]


@pytest.mark.parametrize("case", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_planted_mistake_fails_a_pin(case, monkeypatch):
    _, module, name, mutant, pins = case
    # keep the original reachable for mutants that wrap it
    monkeypatch.setitem(module.__dict__, "_orig_" + name, module.__dict__[name])
    monkeypatch.setattr(module, name, mutant)
    caught = 0
    for pin in pins():
        try:
            pin()
        except Exception:  # an assertion, or a shape error the mistake causes
            caught += 1
    assert caught > 0, "no pin caught the planted mistake"


def test_the_pins_pass_without_a_mistake():
    for pins in (_pins_dense_rmsnorm, _pins_dense_linear, _pins_quant, _pins_routing, _pins_ffn,
                 _pins_hscale,
                 _pins_formats, _pins_tile_map, _pins_gemm, _pins_mx):
        for pin in pins():
            pin()
