"""The per-expert decomposition the full-size GPU tests use (tests/_oracle_pool.py) reproduces the
whole-batch oracle (CPU only): the expert tasks' contributions add up to moe_ffn's output, and
their h maxima and clipping counts to those of moe_ffn's intermediate over every real row."""

import numpy as np

from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_weight_expert, gen_x
from tests import _oracle_pool as P


def test_expert_tasks_add_up_to_the_whole_ffn():
    cfg = CONFIGS["tiny"]
    x = gen_x(cfg).float().numpy()
    lg = gen_logits(cfg).numpy()
    w1f = np.stack([gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H).float().numpy()
                    for e in range(cfg.E)])
    w2f = np.stack([gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I).float().numpy()
                    for e in range(cfg.E)])
    ids, w = R.route_topk(lg, cfg.k)
    ids[5] = -1  # a fully dropped token
    gs_x = Q.global_scale(x)
    gs_h = np.float32(0.05)  # small enough that some h blocks underflow
    whole = M.moe_ffn(x, None, cfg.k, M.QuantWeights.from_float(w1f),
                      M.QuantWeights.from_float(w2f), gs_h, ids=ids, weights=w, keep=True)
    real = whole["perm"]["row_token"] >= 0
    out = np.zeros_like(whole["out"])
    h_max, sat, under = np.float32(0), 0, 0
    for e in range(cfg.E):
        tok = np.nonzero((ids == e).any(axis=1))[0]
        jobs = {"b": (tok, x[tok], ids[tok], w[tok], gs_x, gs_h)}
        _, res = P.expert_task((cfg.E, e, w1f[e], w2f[e], jobs))
        if "b" not in res:
            continue
        t, contrib, hm, (ns, nu) = res["b"]
        out[t] += contrib
        h_max = max(h_max, hm)
        sat, under = sat + ns, under + nu
    assert np.allclose(out, whole["out"], rtol=1e-13, atol=1e-15 * np.abs(whole["out"]).max())
    assert np.all(out[5] == 0)
    assert h_max == np.max(np.abs(whole["h32"][real]))
    assert (sat, under) == Q.block_scale_clipping(whole["h32"][real], gs_h)
    assert under > 0
