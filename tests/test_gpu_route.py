"""GPU parity: moe_permute (top-k softmax routing + expert-bucketed rows) against the oracle.
Ids, offsets and the row map are compared exactly; weights to float32 accuracy."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import routing as R
from synth import CONFIGS, gen_logits
from tests._gpu_util import DEV, to_dev

pytestmark = pytest.mark.gpu


def _compare(p, ids_ref, w_ref, E, k):
    torch.cuda.synchronize()
    T = ids_ref.shape[0]
    pr = R.permute(ids_ref, w_ref, E)
    assert np.array_equal(p["ids"].cpu().numpy(), ids_ref)
    assert np.allclose(p["weights"].cpu().numpy(), w_ref, rtol=2e-6, atol=1e-7)
    assert np.array_equal(p["offs"].cpu().numpy(), pr["offs"])
    assert np.array_equal(p["dst_row"].cpu().numpy().reshape(T, k), pr["dst_row"])
    Rm = p["R_max"]
    rs = p["row_slot"].cpu().numpy()[:Rm]
    rw = p["row_w"].cpu().numpy()[:Rm]
    n = pr["R"]
    assert np.array_equal(rs[:n], pr["row_slot"])
    assert np.all(rs[n:] == -1) and np.all(rw[n:] == 0)
    assert np.allclose(rw[:n], pr["row_w"], rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["tiny", "decode", "mid", "prefill"])
def test_route_configs(name):
    cfg = CONFIGS[name]
    lg = gen_logits(cfg)
    p = nv.permute(lg.to(DEV), cfg.k)
    ids_ref, w_ref = R.route_topk(lg.numpy(), cfg.k)
    _compare(p, ids_ref, w_ref, cfg.E, cfg.k)
    if name == "mid":  # the masked experts are empty
        assert (np.diff(p["offs"].cpu().numpy()) == 0).sum() >= 8


def test_route_no_renormalize_and_ties():
    lg = torch.tensor([[1.0, 3.0, 3.0, 0.0, 3.0], [0.0] * 5, [-np.inf, 2.0, -np.inf, -np.inf, 1.0]],
                      dtype=torch.float32)
    p = nv.permute(lg.to(DEV), 3, renormalize=False)
    ids_ref, w_ref = R.route_topk(lg.numpy(), 3, renormalize=False)
    _compare(p, ids_ref, w_ref, 5, 3)


def test_route_given_ids_with_dropped_slots():
    rng = np.random.default_rng(0)
    T, E, k = 300, 16, 4
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    ids[rng.random((T, k)) < 0.2] = -1
    w = rng.random((T, k)).astype(np.float32)
    p = nv.permute(None, k, ids=to_dev(ids), weights=to_dev(w), E=E)
    _compare(p, ids, w, E, k)


def test_route_empty_batch():
    lg = torch.zeros(0, 8, dtype=torch.float32, device=DEV)
    p = nv.permute(lg, 2)
    torch.cuda.synchronize()
    assert p["offs"].cpu().tolist() == [0] * 9 and p["R_max"] == 0


def test_permute_without_workspace_matches_multi_cta():
    """From 4096 slots the row map is built by many CTAs through the workspace; without one, a
    single CTA builds it.  Both must give the same map."""
    from nvfp4_block_scaled_gsa_b200._native import call, lib
    cfg = CONFIGS["mid"]
    lg = gen_logits(cfg).to(DEV)
    a = nv.permute(lg, cfg.k)
    assert lib().moe_permute_workspace_size(cfg.T, cfg.E, cfg.k) > 0
    T, E, k = cfg.T, cfg.E, cfg.k
    R = a["R_max"]
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    offs = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    dst = torch.empty(T * k, dtype=torch.int32, device=DEV)
    rs = torch.empty(R, dtype=torch.int32, device=DEV)
    rw = torch.empty(R, dtype=torch.float32, device=DEV)
    call("moe_permute", lg.data_ptr(), T, E, k, 1, ids.data_ptr(), w.data_ptr(), offs.data_ptr(),
         dst.data_ptr(), rs.data_ptr(), rw.data_ptr(), None, 0, None,
         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    # the single CTA also takes the top-k itself
    assert torch.equal(ids, a["ids"]) and torch.equal(w, a["weights"])
    assert torch.equal(offs, a["offs"]) and torch.equal(dst, a["dst_row"])
    assert torch.equal(rs, a["row_slot"]) and torch.equal(rw, a["row_w"])


@pytest.mark.parametrize("T,E,k", [(511, 256, 8), (4095, 64, 1), (100, 7, 7)])
def test_route_one_launch_below_the_multi_cta_size(T, E, k):
    """Below 4096 slots one CTA takes the top-k of every token (one warp per token, many tokens
    per warp here) and then builds the row map."""
    rng = np.random.default_rng(T + E + k)
    lg = torch.from_numpy(rng.standard_normal((T, E)).astype(np.float32))
    lg[rng.random((T, E)) < 0.05] = -np.inf  # some experts masked per token
    p = nv.permute(lg.to(DEV), k)
    ids_ref, w_ref = R.route_topk(lg.numpy(), k)
    _compare(p, ids_ref, w_ref, E, k)
