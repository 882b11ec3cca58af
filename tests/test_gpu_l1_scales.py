"""GPU checks of the L1 epilogue's scaling and of what it records about the intermediate h.

* Experts whose weights differ by large, non-power-of-two factors (so their global scales
  gs_w1[e] differ) and activations far from unit scale (gs_x far from 1): the FP32 h values the
  fused epilogue computes (alpha = 1/(gs_x * gs_w1[e]) applied per expert, SwiGLU) match the
  oracle's h32 to the GEMM-stage tolerance, expert by expert; the re-quantized codes pass the
  0.1% bar.  A wrong per-expert alpha or a dropped gs_x moves whole segments and fails both.
* h_stats: the amax of h is bitwise the maximum of the kernel's own h32 over real rows, and the
  clipping counts are exactly the oracle's count rule applied to the kernel's h32.
* Delayed scaling through moe_ffn_forward_ex: the scale left for the next call is the oracle's
  2688 / amax rule applied to the recorded amax, bit for bit, and the next call's output matches
  the oracle run with that scale.
"""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x
from tests._gpu_util import (DEV, compare_requant, cosine, download_nvfp4, rel_fro, to_dev,
                             upload_nvfp4, upload_weights)

pytestmark = pytest.mark.gpu

FACTORS = [0.3, 3.7, 0.55, 1.9, 7.1, 0.21]   # per-expert weight scale (non-powers of two)
X_SCALE = 37.3                               # gs_x = 2688 / amax(x) ~ 16, far from 1


def _scaled_setup(T=200, H=512, I=256, k=3, factors=FACTORS, seed=0, x_scale=X_SCALE):
    E = len(factors)
    cfg = CONFIGS["tiny"]
    x = (gen_x(cfg, T=T, H=H).float().numpy() * np.float32(x_scale)).astype(np.float32)
    lg = torch.randn(T, E, generator=torch.Generator().manual_seed(seed + 5)).numpy()
    ids, w = R.route_topk(lg, k)
    w1f = np.stack([gen_weight_expert(seed, 1, e, 2 * I, H).float().numpy() * f
                    for e, f in enumerate(factors)]).astype(np.float32)
    w2f = np.stack([gen_weight_expert(seed, 2, e, H, I).float().numpy()
                    for e in range(E)]).astype(np.float32)
    w1, w2 = M.QuantWeights.from_float(w1f), M.QuantWeights.from_float(w2f)
    return x, lg, ids, w.astype(np.float32), w1, w2


def _l1_on_oracle_operands(x, ids, w, w1, w2, gs_h, I):
    ref = M.moe_ffn(x, None, ids.shape[1], w1, w2, gs_h, ids=ids, weights=w.astype(np.float64),
                    keep=True)
    perm = ref["perm"]
    Rr, H = perm["R"], x.shape[1]
    valid = perm["row_token"] >= 0
    xc = np.zeros((Rr, H), np.uint8)
    xsf = np.zeros((Rr, H // 16), np.uint8)
    xc[valid] = ref["x_codes"][perm["row_token"][valid]]
    xsf[valid] = ref["x_sf"][perm["row_token"][valid]]
    a, asf = upload_nvfp4(xc, xsf)
    gs_x = to_dev(np.array([ref["gs_x"]], np.float32))
    offs = to_dev(perm["offs"].astype(np.int32))
    row_slot = to_dev(perm["row_slot"].astype(np.int32))
    w1d = upload_weights(w1, w1=True)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    h, sfh, stats, h32 = nv.l1_swiglu_q_stats(a, asf, gs_x, w1d, offs,
                                              to_dev(np.array([gs_h], np.float32)),
                                              row_slot=row_slot, want_h32=True, status=status)
    code, rc = nv.read_status(status)
    assert code == 0 and rc == 0
    hc, hs = download_nvfp4(h, sfh, Rr, I)
    return ref, perm, valid, hc, hs, stats.cpu().numpy().view(np.uint32), h32.cpu().numpy()


def test_l1_distinct_expert_scales_h32_and_codes():
    I = 256
    x, lg, ids, w, w1, w2 = _scaled_setup(I=I)
    assert np.ptp(np.log2(w1.gs)) > 4                 # global scales span > 16x
    assert not np.all(np.log2(w1.gs) == np.round(np.log2(w1.gs)))
    gs_h = np.float32(0.03)
    ref, perm, valid, hc, hs, stats, h32 = _l1_on_oracle_operands(x, ids, w, w1, w2, gs_h, I)
    assert abs(np.log2(ref["gs_x"])) > 3                 # gs_x far from 1
    # FP32 h before quantization, expert by expert, at the GEMM-stage tolerance
    offs = perm["offs"]
    for e in range(w1.E):
        seg = np.zeros_like(valid)
        seg[offs[e]:offs[e + 1]] = True
        seg &= valid
        if seg.any():
            assert rel_fro(h32[seg], ref["h32"][seg]) <= 1e-5, f"expert {e}"
    assert rel_fro(h32[valid], ref["h32"][valid]) <= 1e-5
    frac, far = compare_requant(hc[valid], hs[valid], ref["h_codes"][valid], ref["h_sf"][valid],
                                gs_h)
    assert far == 0 and frac <= 1e-3
    # the statistics: amax bitwise the max of the kernel's own h32, counts by the oracle's rule
    assert stats[0] == np.max(np.abs(h32[valid])).view(np.uint32)
    assert abs(float(stats[0].view(np.float32)) - float(np.max(np.abs(ref["h32"][valid])))) <= \
        1e-5 * float(np.max(np.abs(ref["h32"][valid])))
    assert tuple(int(v) for v in stats[1:]) == Q.block_scale_clipping(h32[valid], gs_h)


@pytest.mark.parametrize("gs_h", [8.0, 1e-4])
def test_l1_clipping_counters(gs_h):
    """A static scale far too large saturates the big experts' block scales; far too small, it
    underflows the small experts' blocks to zero.  The counters follow the oracle's rule on the
    kernel's own h32 exactly, and the oracle's h32 to within boundary cases."""
    I = 256
    factors = [0.001, 3.7, 0.55, 9.0, 0.02, 1.0]
    x, lg, ids, w, w1, w2 = _scaled_setup(I=I, factors=factors)
    ref, perm, valid, hc, hs, stats, h32 = _l1_on_oracle_operands(x, ids, w, w1, w2,
                                                                  np.float32(gs_h), I)
    got = tuple(int(v) for v in stats[1:])
    assert got == Q.block_scale_clipping(h32[valid], np.float32(gs_h))
    want = Q.block_scale_clipping(ref["h32"][valid], np.float32(gs_h))
    nblocks = int(valid.sum()) * I // 16
    assert abs(got[0] - want[0]) <= max(2, nblocks // 1000)
    assert abs(got[1] - want[1]) <= max(2, nblocks // 1000)
    assert (got[0] > 0) if gs_h > 1 else (got[1] > 0)


def test_scale_from_amax_matches_the_oracle_rule():
    vals = np.array([2688.0, 3.0, 1e-30, 0.0, np.inf, np.nan, 7.25, 1e30, 2.0 ** -126],
                    np.float32)
    for v in vals:
        bits = torch.tensor([int(np.float32(v).view(np.uint32).astype(np.int64))],
                            dtype=torch.int64).to(torch.int32).to(DEV)
        gs = torch.zeros(1, dtype=torch.float32, device=DEV)
        nv.scale_from_amax(bits, gs)
        got = gs.cpu().numpy()[0]
        assert got.view(np.uint32) == Q.scale_from_amax(v).view(np.uint32), v


def test_delayed_scale_through_the_ffn():
    """Two calls on one batch with gs_h_delayed = 1: the first quantizes h at the given scale and
    leaves 2688 / amax(h) for the second; the second, on the same batch, uses it (so its h is
    quantized at its own dynamic scale) and leaves the same scale again."""
    cfg = CONFIGS["tiny"]
    x, lg = gen_x(cfg), gen_logits(cfg)
    w1f = np.stack([gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H).float().numpy()
                    for e in range(cfg.E)])
    w2f = np.stack([gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I).float().numpy()
                    for e in range(cfg.E)])
    w1, w2 = M.QuantWeights.from_float(w1f), M.QuantWeights.from_float(w2f)
    w1d, w2d = upload_weights(w1, w1=True), upload_weights(w2)
    gs_h = torch.tensor([64.0], dtype=torch.float32, device=DEV)
    stats = torch.zeros(3, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    xd, lgd = x.to(DEV), lg.to(DEV)
    xs = x.float().numpy()
    outs, scales, amaxes = [], [], []
    for _ in range(2):
        used = gs_h.cpu().numpy()[0]
        out = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1d, w2d, gs_h, delayed=True, h_stats=stats,
                                    status=status)
        code, rc = nv.read_status(status)
        assert code == 0 and rc == 0
        st = stats.cpu().numpy().view(np.uint32)
        amax = st[0].view(np.float32)
        left = gs_h.cpu().numpy()[0]
        assert left.view(np.uint32) == Q.scale_from_amax(amax).view(np.uint32)
        ref = M.moe_ffn(xs, lg.numpy(), cfg.k, w1, w2, np.float32(used), keep=True)
        real = ref["perm"]["row_token"] >= 0
        oracle_amax = np.max(np.abs(ref["h32"][real]))
        assert abs(float(amax) - float(oracle_amax)) <= 1e-5 * float(oracle_amax)
        got = out.float().cpu().numpy().astype(np.float64)
        want = M.bf16_round(ref["out"])
        assert rel_fro(got, want) <= 1e-3 and cosine(got, want) >= 0.9999
        outs.append(got)
        scales.append(left)
        amaxes.append(amax)
    assert amaxes[0] == amaxes[1] and scales[0] == scales[1]
    # the first call's static 64 and the delayed scale differ: the second output is a different
    # quantization of h, not a repeat of the first
    assert scales[0] != np.float32(64.0)
