"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in the oracle (a wrong formula put in place of an oracle function
for the duration of the test) and runs the pins that guard that function: at least one of them
has to fail.  This checks the pins, not the oracle; the oracle itself is never edited.
"""

import numpy as np
import pytest

from oracle import dense as D
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from tests import test_oracle_dense as PD
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


def _pins_routing():
    return [PR.test_topk_matches_bruteforce_subsets_on_tiny,
            PR.test_topk_ties_go_to_lower_id_and_no_renorm,
            PR.test_permute_offsets_order_and_padding]


def _pins_ffn():
    tiny = PR._tiny_inputs()
    return [PR.test_silu_closed_forms, lambda: PR.test_top1_weight1_is_plain_expert_ffn(tiny)]


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
    ("routing: weights not renormalized over the k", R, "route_topk",
     _route_without_renormalization, _pins_routing),
    ("permutation: tokens in descending order inside an expert", R, "permute",
     _permute_descending_tokens, _pins_routing),
    ("SwiGLU: sigmoid(g) in place of silu(g)", M, "silu", _silu_is_sigmoid, _pins_ffn),
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
    for pins in (_pins_dense_rmsnorm, _pins_dense_linear, _pins_quant, _pins_routing, _pins_ffn):
        for pin in pins():
            pin()
