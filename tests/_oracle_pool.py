"""Oracle work for the full-size GPU parity tests, shaped for a spawn-started process pool.

The functions here import only numpy and the oracle, so a worker process never touches CUDA.
Each task carries one expert's float weights (copied back from the device, where the E=256
weight set is drawn) and the rows of every batch that route to it; the worker pre-packs the
expert once with the oracle's quantizer and evaluates the oracle FFN on those rows alone, with
every other slot of the sub-batch dropped, so the result is exactly that expert's weighted
contribution to each of its tokens.
"""

import numpy as np

from oracle import moe as M
from oracle import quant as Q


def limit_blas_threads():
    """Pool initializer: one BLAS thread per worker (the pool supplies the parallelism)."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # threadpoolctl missing: BLAS keeps its default
        pass


class OneExpert:
    """QuantWeights of a single expert `e` standing in for an E-expert set."""

    def __init__(self, E, e, q):
        self.E, self.e, self.q, self.N = E, e, q, q.N

    def dequant(self, e):
        assert e == self.e, "only the expert of this task is evaluated"
        return self.q.dequant(0)


def expert_task(task):
    """task = (E, e, w1 float32 (2I, H), w2 float32 (H, I), jobs) with jobs = {name: (tokens,
    x rows float32 (m, H), ids (m, k), weights (m, k), gs_x, gs_h)}.

    Returns (e, {name: (tokens, contribution float64 (m, H), max|h32| float32, (saturated,
    underflowed) block scales of h)})."""
    E, e, w1f, w2f, jobs = task
    W1 = OneExpert(E, e, M.QuantWeights.from_float(w1f[None]))
    W2 = OneExpert(E, e, M.QuantWeights.from_float(w2f[None]))
    res = {}
    for name, (tokens, x, ids, w, gs_x, gs_h) in jobs.items():
        if len(tokens) == 0:
            continue
        only_e = np.where(ids == e, ids, -1).astype(np.int32)
        r = M.moe_ffn(x, None, ids.shape[1], W1, W2, np.float32(gs_h), ids=only_e, weights=w,
                      gs_x=np.float32(gs_x), keep=True)
        real = r["perm"]["row_token"] >= 0
        h32 = r["h32"][real]
        res[name] = (tokens, r["out"], np.float32(np.max(np.abs(h32))),
                     Q.block_scale_clipping(h32, np.float32(gs_h)))
    return e, res


def group_rows_task(task):
    """task = (g, b float32 (N, K), a rows float32 (n, K), gs_a): the oracle's plain grouped GEMM
    on sampled rows of group g, A quantized with the whole A's global scale.  Returns (g, float64
    (n, N))."""
    g, bf, a, gs_a = task
    q = M.QuantWeights.from_float(bf[None])
    c, s = Q.quantize(a, np.float32(gs_a))
    return g, Q.dequantize(c, s, np.float32(gs_a)) @ q.dequant(0).T
