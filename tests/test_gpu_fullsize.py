"""Parity at the full workload sizes, through moe_ffn_forward (the kernels bench.py times):
decode, mid-batch and prefill batches run whole on the GPU; sampled tokens are checked against
the oracle.  A token's output depends on the rest of the batch only through the activations'
global scale, which the oracle takes from the whole batch."""

import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x
from tests._gpu_util import DEV, cosine, rel_fro

pytestmark = pytest.mark.gpu


class _Sparse:
    def __init__(self, E, N, parts):
        self.E, self.N, self.parts = E, N, parts

    def dequant(self, e):
        return self.parts[e].dequant(0)


@pytest.fixture(scope="module")
def pool():
    ctx = mp.get_context("spawn")  # never fork a process that has a CUDA context
    with ctx.Pool(min(8, os.cpu_count() or 1)) as p:
        yield p


@pytest.mark.parametrize("name,tok", [("decode", 0), ("mid", 5), ("prefill", 8191)])
def test_ffn_full_size_sampled_token(name, tok, pool):
    cfg = CONFIGS[name]
    x, lg = gen_x(cfg), gen_logits(cfg)
    w1 = nv.quantize_w1(lambda e: gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H, device=DEV),
                        cfg.E, cfg.I, cfg.H, device=DEV)
    w2 = nv.quantize_weights(lambda e: gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I, device=DEV),
                             cfg.E, cfg.H, cfg.I, device=DEV)
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = nv.moe_ffn_forward(x.to(DEV), lg.to(DEV), cfg.k, w1, w2, gs_h, status=status)
    code, rc = nv.read_status(status)
    assert code == 0 and rc == 0
    got = out[tok:tok + 1].float().cpu().numpy().astype(np.float64)

    xs = x.float().numpy()
    lgs = lg.numpy()[tok:tok + 1]
    ids, _ = R.route_topk(lgs, cfg.k)
    experts = sorted(int(e) for e in set(ids.ravel()) if e >= 0)
    w1f = [gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H, device=DEV).float().cpu().numpy()
           for e in experts]
    w2f = [gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I, device=DEV).float().cpu().numpy()
           for e in experts]
    # the oracle's weight pre-pack of each expert, in worker processes
    q1 = pool.map(M.QuantWeights.from_float, [w[None] for w in w1f])
    q2 = pool.map(M.QuantWeights.from_float, [w[None] for w in w2f])
    W1 = _Sparse(cfg.E, 2 * cfg.I, dict(zip(experts, q1)))
    W2 = _Sparse(cfg.E, cfg.H, dict(zip(experts, q2)))
    ref = M.moe_ffn(xs[tok:tok + 1], lgs, cfg.k, W1, W2, np.float32(cfg.gs_h),
                    experts=experts, gs_x=Q.global_scale(xs))["out"]
    want = M.bf16_round(ref)
    assert rel_fro(got, want) <= 1e-3
    assert cosine(got, want) >= 0.9999
