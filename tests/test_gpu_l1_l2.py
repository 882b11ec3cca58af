"""GPU parity for the two fused grouped GEMMs on identical quantized operands:

* L1 + SwiGLU + NVFP4 re-quantization: h codes may differ by one E2M1 step on at most 0.1% of
  the elements (a block whose scale byte differs counts whole);
* L2 + routing weight + scatter to token order: FP32 result within relative Frobenius 1e-5 of
  the oracle.
"""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x
from tests._gpu_util import (DEV, compare_requant, download_nvfp4, rel_fro, to_dev, upload_nvfp4,
                             upload_weights)

pytestmark = pytest.mark.gpu


def _weights(seed, which, E, N, K):
    wf = np.stack([gen_weight_expert(seed, which, e, N, K).float().numpy() for e in range(E)])
    w = M.QuantWeights.from_float(wf)
    return w, upload_weights(w, w1=(which == 1))


def _setup(T, H, I, E, k, seed=0, drop=0.0):
    cfg = CONFIGS["tiny"]
    x = gen_x(cfg, T=T, H=H).float().numpy()
    lg = torch.randn(T, E, generator=torch.Generator().manual_seed(seed + 3)).numpy()
    ids, w = R.route_topk(lg, k)
    if drop:
        rng = np.random.default_rng(seed)
        ids = np.where(rng.random(ids.shape) < drop, -1, ids).astype(np.int32)
    w32 = w.astype(np.float32)
    w1, w1d = _weights(seed, 1, E, 2 * I, H)
    w2, w2d = _weights(seed, 2, E, H, I)
    return x, ids, w32, w1, w1d, w2, w2d


@pytest.mark.parametrize("T,H,I,E,k", [
    (64, 256, 128, 8, 2), (200, 512, 256, 6, 3), (33, 7168, 2048, 2, 2), (96, 256, 128, 256, 8),
    # decode-like batches (few tokens per expert)
    (16, 256, 128, 8, 2), (32, 512, 256, 6, 3), (20, 7168, 2048, 3, 2), (16, 256, 128, 256, 8),
    (1, 256, 128, 4, 1),
    # 128+ rows per expert (several M-tiles per expert; from 32 rows per expert the FFN adds
    # into token rows)
    (640, 256, 128, 4, 2), (640, 1024, 512, 2, 1),
    # 1024+ rows per expert: 256-row tiles on CTA pairs (odd block counts: half-empty pair tiles)
    (2304, 256, 128, 2, 1)])
def test_l1_and_l2_match_oracle(T, H, I, E, k):
    x, ids, w32, w1, w1d, w2, w2d = _setup(T, H, I, E, k, drop=0.1)
    gs_h = np.float32(64.0 if H <= 512 else 1.0)
    ref = M.moe_ffn(x, None, k, w1, w2, gs_h, ids=ids, weights=w32.astype(np.float64), keep=True)
    perm = ref["perm"]
    Rr = perm["R"]
    valid = perm["row_token"] >= 0
    # identical quantized operands: the oracle's permuted x codes
    xc = np.zeros((Rr, H), np.uint8)
    xsf = np.zeros((Rr, H // 16), np.uint8)
    xc[valid] = ref["x_codes"][perm["row_token"][valid]]
    xsf[valid] = ref["x_sf"][perm["row_token"][valid]]
    a, asf = upload_nvfp4(xc, xsf)
    gs_x = to_dev(np.array([ref["gs_x"]], np.float32))
    offs = to_dev(perm["offs"].astype(np.int32))
    gs_h_d = to_dev(np.array([gs_h], np.float32))

    # ---- L1 GEMM stage on its own (plain epilogue, FP32) within 1e-5
    c1 = nv.grouped_gemm(a, asf, gs_x, w1d, offs, out_dtype=torch.float32)
    # ---- L1 fused SwiGLU + re-quantization (every row; and with the row map, which skips
    # all-padding row groups but must give the same bytes on real rows)
    h, sfh = nv.l1_swiglu_q(a, asf, gs_x, w1d, offs, gs_h_d)
    row_slot = to_dev(perm["row_slot"].astype(np.int32))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    h2, sfh2 = nv.l1_swiglu_q(a, asf, gs_x, w1d, offs, gs_h_d, row_slot=row_slot, status=status)
    torch.cuda.synchronize()
    hc2, hs2 = download_nvfp4(h2, sfh2, Rr, I)
    c1_logical = c1.cpu().numpy()[:, nv.w1_row_map(I).numpy()]  # stored -> logical columns
    assert rel_fro(c1_logical[valid], ref["c1"][valid]) <= 1e-5
    hc, hs = download_nvfp4(h, sfh, Rr, I)
    frac, far = compare_requant(hc[valid], hs[valid], ref["h_codes"][valid], ref["h_sf"][valid], gs_h)
    assert far == 0
    assert frac <= 1e-3
    # the row-map call (padding row groups skipped) against the oracle too
    frac2, far2 = compare_requant(hc2[valid], hs2[valid], ref["h_codes"][valid], ref["h_sf"][valid],
                                  gs_h)
    assert far2 == 0 and frac2 <= 1e-3
    # same kernel, same accumulation order: identical bytes on real rows
    assert np.array_equal(hc2[valid], hc[valid]) and np.array_equal(hs2[valid], hs[valid])

    # ---- L2 + scatter on the oracle's h codes (identical operands)
    h_o, sfh_o = upload_nvfp4(ref["h_codes"], ref["h_sf"])
    row_w = to_dev(perm["row_w"].astype(np.float32))
    dst_row = to_dev(perm["dst_row"].reshape(-1).astype(np.int32))
    acc, out = nv.l2_scatter(h_o, sfh_o, gs_h_d, w2d, offs, row_slot, row_w, dst_row, T, k,
                             status=status)
    torch.cuda.synchronize()
    code, rc = nv.read_status(status)
    assert code == 0 and rc == 0
    assert rel_fro(acc.cpu().numpy(), ref["out"]) <= 1e-5
    assert torch.equal(out.cpu(), acc.cpu().to(torch.bfloat16))
    dropped = np.all(ids < 0, axis=1)
    assert np.all(acc.cpu().numpy()[dropped] == 0)
    # the scatter-ADD form (rows added into token rows as tiles are produced, N-slice-major):
    # the same FP32 sum up to addition order
    acc2, out2 = nv.l2_scatter_add(h_o, sfh_o, gs_h_d, w2d, offs, row_slot, row_w, dst_row, T, k,
                                   status=status)
    torch.cuda.synchronize()
    code, rc = nv.read_status(status)
    assert code == 0 and rc == 0
    assert rel_fro(acc2.cpu().numpy(), ref["out"]) <= 1e-5
    assert torch.equal(out2.cpu(), acc2.cpu().to(torch.bfloat16))
    assert np.all(acc2.cpu().numpy()[dropped] == 0)


def test_l2_bad_row_slot_is_flagged():
    x, ids, w32, w1, w1d, w2, w2d = _setup(16, 256, 128, 2, 1)
    perm = R.permute(ids, w32, 2)
    Rr = perm["R"]
    h = torch.zeros(Rr, 64, dtype=torch.uint8, device=DEV)
    sfh = torch.zeros(nv.sf_bytes(Rr, 128), dtype=torch.uint8, device=DEV)
    rs = perm["row_slot"].astype(np.int32).copy()
    rs[0] = 999  # out of range slot (T*k = 16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    nv.l2_scatter(h, sfh, torch.ones(1, device=DEV), w2d, to_dev(perm["offs"].astype(np.int32)),
                  to_dev(rs), to_dev(perm["row_w"].astype(np.float32)),
                  to_dev(perm["dst_row"].reshape(-1).astype(np.int32)), 16, 1, status=status)
    code, rc = nv.read_status(status)
    assert code & 2 and rc == 7
    # the scatter-add form flags (and skips) the same bad slot
    status.zero_()
    nv.l2_scatter_add(h, sfh, torch.ones(1, device=DEV), w2d,
                      to_dev(perm["offs"].astype(np.int32)), to_dev(rs),
                      to_dev(perm["row_w"].astype(np.float32)),
                      to_dev(perm["dst_row"].reshape(-1).astype(np.int32)), 16, 1, status=status)
    code, rc = nv.read_status(status)
    assert code & 2 and rc == 7
