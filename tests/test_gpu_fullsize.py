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


def test_grouped_gemm_sweep_full_size_sampled_rows(pool):
    """The standalone grouped GEMM at the sweep shape (E=32, M_g ~ U{0..4096}, K=7168, N=4096,
    bf16 out, pair tiles): rows sampled from two groups against the oracle, which quantizes those
    rows itself with the global scale of the whole A (from its amax, taken on the host)."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    cfg = CONFIGS["sweep"]
    m, offs, a, w = bench.sweep_operands(cfg, DEV)
    codes, sf, gs = nv.quantize(a)
    out = nv.grouped_gemm(codes, sf, gs, w, offs, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    a_cpu = a.cpu()
    gs_ref = Q.global_scale(np.array([[float(a_cpu.abs().max())]], np.float32))
    order = np.argsort(m)
    groups = [int(order[-1]), int(order[len(order) // 2])]  # the largest and a middle-sized one
    wf = [gen_weight_expert(cfg.seed, 1, g, cfg.N, cfg.K, device=DEV).float().cpu().numpy()
          for g in groups]
    qw = pool.map(M.QuantWeights.from_float, [x[None] for x in wf])
    offs_h = offs.cpu().numpy()
    for g, q in zip(groups, qw):
        rows = offs_h[g] + np.array([0, m[g] // 2, m[g] - 1])
        xr = a_cpu[rows].float().numpy()
        c, s = Q.quantize(xr, gs_ref)
        ref = Q.dequantize(c, s, gs_ref) @ q.dequant(0).T
        got = out[torch.as_tensor(rows, device=DEV)].float().cpu().numpy().astype(np.float64)
        want = M.bf16_round(ref)
        assert rel_fro(got, want) <= 1e-3
        assert cosine(got, want) >= 0.9999
