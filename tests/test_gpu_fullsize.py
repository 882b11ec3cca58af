"""Parity at the full workload sizes, in the launch configuration bench.py times.

The decode (T=16), mid-batch (T=512, Zipf-skewed with empty experts, x outliers) and prefill
(T=8192) batches run whole through moe_ffn_forward_ex on the shared E=256 weight set, and EVERY
output row is compared with the oracle's float64 result rounded once to bf16: relative Frobenius
<= 1e-3 and cosine >= 0.9999 over the batch; per token, cosine >= 0.9999, relative Frobenius
<= 2e-2, and at most 2% of the tokens above 1e-3 (the reason is in the test).  The oracle runs
expert by expert in a spawn-started process pool (tests/_oracle_pool.py): each task pre-packs one
expert and evaluates every batch's rows that route to it.  The same pass gives the oracle's amax
of the intermediate h and its block-scale clipping counts, checked against the kernel's h_stats.

The standalone grouped GEMM runs at the sweep shape (E=32 groups, K=7168, N=4096, pair tiles) and
is checked on the first, the last and ten random rows of every non-empty group.
"""

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
from tests import _oracle_pool as P
from tests._gpu_util import DEV, cosine, rel_fro

pytestmark = pytest.mark.gpu

NAMES = ("decode", "mid", "prefill")


def _workers():
    return max(2, min(16, os.cpu_count() or 2))


@pytest.fixture(scope="module")
def pool():
    ctx = mp.get_context("spawn")  # never fork a process that has a CUDA context
    with ctx.Pool(_workers(), initializer=P.limit_blas_threads) as p:
        yield p


@pytest.fixture(scope="module")
def runs(pool):
    """GPU outputs and h statistics of the three batches, and the oracle's, row by row."""
    c0 = CONFIGS["prefill"]
    E, H, I, seed = c0.E, c0.H, c0.I, c0.seed
    for name in NAMES:
        c = CONFIGS[name]
        assert (c.E, c.H, c.I, c.seed) == (E, H, I, seed), "the three batches share one weight set"
    w1 = nv.quantize_w1(lambda e: gen_weight_expert(seed, 1, e, 2 * I, H, device=DEV), E, I, H,
                        device=DEV)
    w2 = nv.quantize_weights(lambda e: gen_weight_expert(seed, 2, e, H, I, device=DEV), E, H, I,
                             device=DEV)
    gpu, inputs = {}, {}
    for name in NAMES:
        cfg = CONFIGS[name]
        x, lg = gen_x(cfg), gen_logits(cfg)
        gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=DEV)
        stats = torch.zeros(3, dtype=torch.int32, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        xd, lgd = x.to(DEV), lg.to(DEV)
        out = nv.moe_ffn_forward(xd, lgd, cfg.k, w1, w2, gs_h, status=status)
        # the statistics are gathered on the slot-ordered path, whose output is reproducible
        det = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1, w2, gs_h, deterministic=True,
                                    status=status)
        det_stats = nv.moe_ffn_forward_ex(xd, lgd, cfg.k, w1, w2, gs_h, deterministic=True,
                                          h_stats=stats, status=status)
        code, rc = nv.read_status(status)
        gpu[name] = dict(out=out.float().cpu().numpy().astype(np.float64),
                         same_as_plain=bool(torch.equal(det, det_stats)), code=code, rc=rc,
                         stats=stats.cpu().numpy().view(np.uint32).copy())
        xs = x.float().numpy()
        ids, w = R.route_topk(lg.numpy(), cfg.k)
        inputs[name] = (xs, ids, w, Q.global_scale(xs), np.float32(cfg.gs_h))
    del w1, w2
    torch.cuda.empty_cache()

    ref = {n: np.zeros((CONFIGS[n].T, H)) for n in NAMES}
    h_max = {n: np.float32(0) for n in NAMES}
    clip = {n: [0, 0] for n in NAMES}
    B = _workers()
    for e0 in range(0, E, B):
        tasks = []
        for e in range(e0, min(E, e0 + B)):
            jobs = {}
            for name in NAMES:
                xs, ids, w, gs_x, gs_h = inputs[name]
                tok = np.nonzero((ids == e).any(axis=1))[0]
                if len(tok):
                    jobs[name] = (tok, xs[tok], ids[tok], w[tok], gs_x, gs_h)
            if not jobs:
                continue
            w1f = gen_weight_expert(seed, 1, e, 2 * I, H, device=DEV).float().cpu().numpy()
            w2f = gen_weight_expert(seed, 2, e, H, I, device=DEV).float().cpu().numpy()
            tasks.append((E, e, w1f, w2f, jobs))
        for _, res in pool.imap_unordered(P.expert_task, tasks):
            for name, (tok, contrib, hm, (ns, nu)) in res.items():
                ref[name][tok] += contrib
                h_max[name] = max(h_max[name], hm)
                clip[name][0] += ns
                clip[name][1] += nu
    return gpu, ref, h_max, clip, inputs


@pytest.mark.parametrize("name", NAMES)
def test_ffn_full_size_every_row(name, runs):
    gpu, ref, _, _, inputs = runs
    g = gpu[name]
    assert g["code"] == 0 and g["rc"] == 0
    got, want = g["out"], M.bf16_round(ref[name])
    assert rel_fro(got, want) <= 1e-3
    assert cosine(got, want) >= 0.9999
    # token by token: a row placed in the wrong token, a late persistent tile or a stale slot
    # gives that token an error of the order of its own size, and stands out here even when the
    # batch-wide figures still pass.  The bound per token is looser than the batch's: the
    # re-quantized intermediate may differ by one E2M1 step on 0.1% of its elements, and one
    # such step on a large element of a slot's h row moves that token's output by up to ~1%.
    ids = inputs[name][1]
    dropped = np.all(ids < 0, axis=1)
    assert np.all(got[dropped] == 0)
    live = np.nonzero(~dropped)[0]
    errs = np.array([rel_fro(got[t], want[t]) for t in live])
    coss = np.array([cosine(got[t], want[t]) for t in live])
    q = np.quantile(errs, [0.5, 0.99, 1.0])
    print(f"{name}: per-token rel_fro median {q[0]:.2e}, p99 {q[1]:.2e}, max {q[2]:.2e}; "
          f"{np.mean(errs > 1e-3):.4f} of tokens above 1e-3; min cosine {coss.min():.6f}")
    assert coss.min() >= 0.9999, live[np.argmin(coss)]
    assert errs.max() <= 2e-2, live[np.argmax(errs)]
    assert np.mean(errs > 1e-3) <= 0.02


@pytest.mark.parametrize("name", NAMES)
def test_ffn_statistics_leave_the_output_unchanged(name, runs):
    """Gathering the h statistics leaves the (slot-ordered, reproducible) output bitwise as it
    is without them."""
    assert runs[0][name]["same_as_plain"]


@pytest.mark.parametrize("name", NAMES)
def test_h_amax_and_clipping_at_full_size(name, runs):
    """The L1 epilogue's amax of h over every real row, against the oracle's: equal to FP32
    accumulation accuracy (the GEMM stage tolerance, 1e-5 relative); its clipping counts equal
    the oracle's to within the blocks whose scale sits on an E4M3 limit (none at these sizes)."""
    gpu, _, h_max, clip, _ = runs
    st = gpu[name]["stats"]
    amax = np.uint32(st[0]).view(np.float32)
    assert amax > 0
    assert abs(float(amax) - float(h_max[name])) <= 1e-5 * float(h_max[name])
    assert abs(int(st[1]) - clip[name][0]) <= 2 and abs(int(st[2]) - clip[name][1]) <= 2
    # at the calibrated static scale nothing clips on these workloads
    assert int(st[1]) == 0 and int(st[2]) == 0


def test_grouped_gemm_sweep_full_size_rows_of_every_group(pool):
    """The standalone grouped GEMM at the sweep shape (E=32, M_g ~ U{0..4096}, K=7168, N=4096,
    bf16 out, pair tiles): the first, the last and ten random rows of every non-empty group
    against the oracle, which quantizes those rows itself with the whole A's global scale."""
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
    offs_h = offs.cpu().numpy()
    rng = np.random.default_rng(0)
    tasks, rows_of = [], {}
    for g in range(cfg.E):
        if m[g] == 0:
            continue
        rows = offs_h[g] + np.unique(np.concatenate(
            [[0, m[g] - 1], rng.integers(0, m[g], size=min(10, m[g]))]))
        rows_of[g] = rows
        bf = gen_weight_expert(cfg.seed, 1, g, cfg.N, cfg.K, device=DEV).float().cpu().numpy()
        tasks.append((g, bf, a_cpu[rows].float().numpy(), gs_ref))
    assert len(tasks) >= 30
    got_all = out.float().cpu().numpy().astype(np.float64)
    for g, ref in pool.imap_unordered(P.group_rows_task, tasks):
        got = got_all[rows_of[g]]
        want = M.bf16_round(ref)
        assert rel_fro(got, want) <= 1e-3, f"group {g}"
        assert cosine(got, want) >= 0.9999, f"group {g}"
