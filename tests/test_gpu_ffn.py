"""GPU parity of the whole expert FFN (moe_ffn_forward) and of the weight pre-pack, against the
oracle: final bf16 output within relative Frobenius 1e-3 and cosine >= 0.9999 of the oracle's
float64 result rounded once to bf16 (the output type; bf16 rounding alone is ~1e-3 relative, so
the comparison is made in the output's own precision)."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import formats as F
from oracle import moe as M
from oracle import quant as Q
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x
from tests._gpu_util import DEV, cosine, rel_fro

pytestmark = pytest.mark.gpu


def _prepack_both(cfg, which, N, K):
    wf = [gen_weight_expert(cfg.seed, which, e, N, K) for e in range(cfg.E)]
    if which == 1:
        wd = nv.quantize_w1(lambda e: wf[e].to(DEV), cfg.E, N // 2, K)
    else:
        wd = nv.quantize_weights(lambda e: wf[e].to(DEV), cfg.E, N, K)
    wo = M.QuantWeights.from_float(np.stack([w.float().numpy() for w in wf]))
    return wd, wo


@pytest.mark.parametrize("which", [1, 2])
def test_weight_prepack_bit_exact(which):
    cfg = CONFIGS["tiny"]
    N, K = (2 * cfg.I, cfg.H) if which == 1 else (cfg.H, cfg.I)
    wd, wo = _prepack_both(cfg, which, N, K)
    torch.cuda.synchronize()
    E = cfg.E
    codes = wd.codes.cpu().numpy().reshape(E, N, K // 2)
    sf = Q.untile_sf(wd.sf.cpu().numpy(), E * N, K // 16).reshape(E, N, K // 16)
    if which == 1:  # stored rows are gate/up interleaved; bring them back to logical order
        m = nv.w1_row_map(cfg.I).numpy()
        codes, sf = codes[:, m], sf[:, m]
    assert np.array_equal(wd.gs.cpu().numpy(), wo.gs)
    assert np.array_equal(codes, wo.codes)
    assert np.array_equal(sf, wo.sf)


def _ffn_check(cfg, x, lg):
    w1d, w1o = _prepack_both(cfg, 1, 2 * cfg.I, cfg.H)
    w2d, w2o = _prepack_both(cfg, 2, cfg.H, cfg.I)
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=DEV)
    out = nv.moe_ffn_forward(x.to(DEV), lg.to(DEV), cfg.k, w1d, w2d, gs_h)
    torch.cuda.synchronize()
    ref = M.moe_ffn(x.float().numpy(), lg.numpy(), cfg.k, w1o, w2o, np.float32(cfg.gs_h))
    got = out.float().cpu().numpy()
    return got, ref


def test_ffn_tiny_end_to_end():
    cfg = CONFIGS["tiny"]
    got, ref = _ffn_check(cfg, gen_x(cfg), gen_logits(cfg))
    want = M.bf16_round(ref["out"])
    assert rel_fro(got, want) <= 1e-3
    assert cosine(got, want) >= 0.9999
    assert rel_fro(got, ref["out"]) <= 3e-3  # unrounded: bf16 rounding dominates


def test_ffn_tokens_with_all_slots_dropped_are_zero():
    cfg = CONFIGS["tiny"]
    lg = gen_logits(cfg)
    lg[5] = float("-inf")
    lg[17] = float("-inf")
    got, ref = _ffn_check(cfg, gen_x(cfg), lg)
    assert np.all(got[5] == 0) and np.all(got[17] == 0)
    assert rel_fro(got, M.bf16_round(ref["out"])) <= 1e-3


def test_ffn_repeatable_and_workspace_reuse():
    cfg = CONFIGS["tiny"]
    x, lg = gen_x(cfg).to(DEV), gen_logits(cfg).to(DEV)
    w1d, _ = _prepack_both(cfg, 1, 2 * cfg.I, cfg.H)
    w2d, _ = _prepack_both(cfg, 2, cfg.H, cfg.I)
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=DEV)
    ws = torch.empty(nv.ffn_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8,
                     device=DEV)
    a = nv.moe_ffn_forward(x, lg, cfg.k, w1d, w2d, gs_h, ws=ws).clone()
    b = nv.moe_ffn_forward(x, lg, cfg.k, w1d, w2d, gs_h, ws=ws)
    torch.cuda.synchronize()
    # FP32 reduction order may differ between runs; the bf16 results agree to rounding
    assert rel_fro(a.float().cpu().numpy(), b.float().cpu().numpy()) <= 1e-3


def test_ffn_rejects_small_workspace():
    cfg = CONFIGS["tiny"]
    x, lg = gen_x(cfg).to(DEV), gen_logits(cfg).to(DEV)
    w1d, _ = _prepack_both(cfg, 1, 2 * cfg.I, cfg.H)
    w2d, _ = _prepack_both(cfg, 2, cfg.H, cfg.I)
    ws = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(nv.Nvfp4Error) as ei:
        nv.moe_ffn_forward(x, lg, cfg.k, w1d, w2d, torch.ones(1, device=DEV), ws=ws)
    assert ei.value.code == 4


@pytest.mark.parametrize("T", [16, 32, 3])
def test_ffn_small_batch_end_to_end(T):
    """Decode-sized batches: a few tokens per expert, most rows of every M-tile padding."""
    from dataclasses import replace
    cfg = replace(CONFIGS["tiny"], T=T)
    got, ref = _ffn_check(cfg, gen_x(cfg), gen_logits(cfg))
    want = M.bf16_round(ref["out"])
    assert rel_fro(got, want) <= 1e-3
    assert cosine(got, want) >= 0.9999


@pytest.mark.parametrize("T", [640, 4096])
def test_ffn_prefill_sized_batch_end_to_end(T):
    """160 / 1024 rows per expert on average: the L2 epilogue stages its rows through shared
    memory; at 1024 both GEMMs also take 256-row tiles on CTA pairs."""
    from dataclasses import replace
    cfg = replace(CONFIGS["tiny"], T=T)
    assert nv.rows_max(cfg.T, cfg.E, cfg.k) >= (1024 if T == 4096 else 256) * cfg.E
    got, ref = _ffn_check(cfg, gen_x(cfg), gen_logits(cfg))
    want = M.bf16_round(ref["out"])
    assert rel_fro(got, want) <= 1e-3
    assert cosine(got, want) >= 0.9999


@pytest.mark.parametrize("T", [640, 4096])
def test_ffn_token_row_reductions_against_slot_ordered_sum(T):
    """From 32 routed rows per expert the FFN adds each slot's weighted row into its token's
    FP32 row as the L2 tiles are produced (order not fixed); NVFP4_FFN_DETERMINISTIC keeps the
    per-slot rows and their slot-ordered sum.  The two differ only by FP32 addition order: at most
    one bf16 step on a small fraction of the outputs.  Fully dropped tokens stay exact zeros in
    both, and both match the oracle."""
    from dataclasses import replace
    cfg = replace(CONFIGS["tiny"], T=T)
    assert T * cfg.k >= 32 * cfg.E
    x, lg = gen_x(cfg), gen_logits(cfg)
    lg[7] = float("-inf")
    lg[T - 1] = float("-inf")
    w1d, w1o = _prepack_both(cfg, 1, 2 * cfg.I, cfg.H)
    w2d, w2o = _prepack_both(cfg, 2, cfg.H, cfg.I)
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=DEV)
    xd, lgd = x.to(DEV), lg.to(DEV)
    fast = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1d, w2d, gs_h).float().cpu().numpy()
    det = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1d, w2d, gs_h,
                                deterministic=True).float().cpu().numpy()
    det2 = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1d, w2d, gs_h,
                                 deterministic=True).float().cpu().numpy()
    plain = nv.moe_ffn_forward(xd, lgd, cfg.k, w1d, w2d, gs_h).float().cpu().numpy()
    assert np.array_equal(det, det2)  # the slot-ordered sum is bitwise reproducible
    for out in (fast, det, plain):
        assert np.all(out[7] == 0) and np.all(out[T - 1] == 0)
    diff = fast != det
    assert diff.mean() <= 0.01
    step = np.abs(det) * 2.0 ** -7 + 1e-30  # one bf16 step (8 significant bits) or less
    assert np.all(np.abs(fast - det)[diff] <= step[diff])
    ref = M.bf16_round(M.moe_ffn(x.float().numpy(), lg.numpy(), cfg.k, w1o, w2o,
                                 np.float32(cfg.gs_h))["out"])
    for out in (fast, det, plain):
        assert rel_fro(out, ref) <= 1e-3 and cosine(out, ref) >= 0.9999
