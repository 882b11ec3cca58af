"""MoE routing and expert-bucketed row permutation (oracle side).

The pages list "the MoE routing logic (top-k selection, slot mapping)" among the pieces the
grouped GEMM does not do ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our
Adaptation"); the grouped GEMM itself is 2D x 3D over tokens bucketed per expert (section
"The Reference Kernel: ScaledGroupedGemmKernel").  Everything below that is more specific
than that is our reading:

* probabilities p = softmax(logits) over the E experts of a token (float64);
* the k experts with the largest logits (softmax is monotonic, so this is the top-k of p,
  decided on the float32 logits exactly); equal logits go to the lower expert id;
* weights w_j = p_j / sum of the k selected p (renormalize=True), or p_j;
* a selected expert whose logit is -inf (a masked expert) gives a dropped slot: id -1,
  weight 0.  With routing given as ids, ids < 0 are dropped slots;
* rows of the permuted activation matrix: experts in ascending id, each expert's segment
  padded to a multiple of 128 rows; inside a segment, slots in ascending token then slot j.
"""

import numpy as np

PAD = 128


def route_topk(logits, k, renormalize=True):
    """Top-k softmax routing.  logits float32 (T, E) -> ids int32 (T, k), w float64 (T, k)."""
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    assert 1 <= k <= E
    ids = np.empty((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    l64 = lg.astype(np.float64)
    for t in range(T):
        # stable sort on -logit keeps the lower id first among equal logits
        order = np.argsort(-l64[t], kind="stable")[:k]
        ids[t] = order
        m = np.max(l64[t])
        if not np.isfinite(m):  # every expert masked
            ids[t] = -1
            continue
        e = np.exp(l64[t] - m)
        p = e / e.sum()
        sel = p[order]
        dropped = ~np.isfinite(l64[t][order])
        sel = np.where(dropped, 0.0, sel)
        ids[t] = np.where(dropped, -1, order)
        if renormalize:
            s = sel.sum()
            w[t] = sel / s if s > 0 else 0.0
        else:
            w[t] = sel
    return ids, w


def permute(ids, w, E):
    """Bucket the T*k slots by expert.

    Returns dict with
      counts  int64 (E,)     tokens routed to each expert (M_e)
      offs    int64 (E+1,)   start row of each expert's 128-padded segment; offs[E] = R
      dst_row int64 (T, k)   permuted row of slot (t, j), -1 for a dropped slot
      row_token int64 (R,)   token of each row, -1 for padding rows
      row_slot  int64 (R,)   slot t*k + j of each row, -1 for padding rows
      row_w   float64 (R,)   routing weight of each row, 0 for padding rows
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if ids[t, j] >= 0:
                counts[ids[t, j]] += 1
    padded = ((counts + PAD - 1) // PAD) * PAD
    offs = np.zeros(E + 1, dtype=np.int64)
    offs[1:] = np.cumsum(padded)
    R = int(offs[E])
    dst_row = np.full((T, k), -1, dtype=np.int64)
    row_token = np.full(R, -1, dtype=np.int64)
    row_slot = np.full(R, -1, dtype=np.int64)
    row_w = np.zeros(R, dtype=np.float64)
    fill = offs[:E].copy()
    for t in range(T):  # ascending token, then ascending slot j
        for j in range(k):
            e = ids[t, j]
            if e < 0:
                continue
            r = fill[e]
            fill[e] += 1
            dst_row[t, j] = r
            row_token[r] = t
            row_slot[r] = t * k + j
            row_w[r] = w[t, j]
    return dict(counts=counts, offs=offs, dst_row=dst_row, row_token=row_token, row_slot=row_slot,
                row_w=row_w, R=R)
