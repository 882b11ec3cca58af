"""Grouped GEMM, SwiGLU, re-quantization and weighted scatter: the whole expert FFN.

The pipeline the pages describe ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", sections "Our
Adaptation" and "Phase 3: Full MoE pipeline"; "May 24, 2026 — Session Start Plan", section 5
"NVFP4-1.1: Fuse FP4 into SwiGLU Epilogue"):

    stage_activation (BF16 -> NVFP4) -> L1 grouped GEMM -> SiLU gate * up -> NVFP4 ->
    L2 grouped GEMM -> scatter with routing weights

Here every GEMM is a float64 matmul of the dequantized operands, one expert at a time
(exact products, float64 sums).  The readings the pages leave open:

* W1 of an expert is (2I, H): rows [0, I) are the gate projection, rows [I, 2I) the up
  projection; h = silu(gate) * up, with no clamp.  The pages' "up_correction" is never defined
  and is not applied (parity unpinned for it).
* h is rounded to float32 and re-quantized to NVFP4 with a given global scale gs_h (a static
  scale: the whole-tensor amax of h is unknown when a fused epilogue writes its first tile).
* out[t] = sum_j w_tj * Y[row(t, j)] in float64; dropped slots contribute nothing.
"""

import math

import numpy as np

from .formats import unpack_nibbles
from .quant import dequantize, global_scale, quantize
from .routing import permute, route_topk


class QuantWeights:
    """Per-expert NVFP4 weights: packed codes (E, N, K/2), logical scales (E, N, K/16),
    global scales (E,).  ``dequant(e)`` gives the float64 (N, K) matrix of expert e."""

    def __init__(self, codes, sf, gs):
        self.codes = codes
        self.sf = sf
        self.gs = np.asarray(gs, dtype=np.float32)

    @property
    def E(self):
        return self.codes.shape[0]

    @property
    def N(self):
        return self.codes.shape[1]

    def dequant(self, e):
        return dequantize(unpack_nibbles(self.codes[e]), self.sf[e], self.gs[e])

    @staticmethod
    def from_float(w):
        """Quantize float (E, N, K) weights expert by expert, each with its own amax scale."""
        w = np.asarray(w, dtype=np.float32)
        E, N, K = w.shape
        codes = np.empty((E, N, K // 2), dtype=np.uint8)
        sf = np.empty((E, N, K // 16), dtype=np.uint8)
        gs = np.empty(E, dtype=np.float32)
        for e in range(E):
            gs[e] = global_scale(w[e])
            c, s = quantize(w[e], gs[e])
            codes[e] = (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)
            sf[e] = s
        return QuantWeights(codes, sf, gs)


def silu(g):
    """SiLU in float64: g / (1 + exp(-g))."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def silu_scalar(g):
    """Scalar SiLU with math.exp, for pins that evaluate single values."""
    try:
        return g / (1.0 + math.exp(-g))
    except OverflowError:
        return -0.0 if g < 0 else 0.0


def grouped_gemm(a, b_dequant, offs, rows_valid=None):
    """2D x 3D grouped GEMM: C[r] = A[r] @ B_e^T for each row r of expert e's segment.

    a          float64 (R, K) dequantized activations, rows bucketed by expert
    b_dequant  callable e -> float64 (N, K)
    offs       (E+1,) segment starts
    rows_valid optional (E,) number of real rows per segment; others are left at 0
    """
    E = len(offs) - 1
    R = int(offs[E])
    out = None
    for e in range(E):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if rows_valid is not None:
            hi = lo + int(rows_valid[e])
        if hi <= lo:
            continue
        b = b_dequant(e)
        if out is None:
            out = np.zeros((R, b.shape[0]), dtype=np.float64)
        out[lo:hi] = a[lo:hi] @ b.T
    return out if out is not None else np.zeros((R, 0))


def moe_ffn(x, logits, k, w1, w2, gs_h, renormalize=True, ids=None, weights=None,
            keep=False, experts=None, gs_x=None):
    """The whole expert FFN, step by step.

    x        (T, H) float (the bf16 activations, as float32)
    logits   (T, E) float32, or None when ``ids``/``weights`` give the routing
    w1, w2   QuantWeights (or any object with E, N and dequant(e)) with N = 2I (gate rows
             then up rows) and N = H
    gs_h     float32 static global scale of the intermediate
    experts  optional iterable restricting which experts are evaluated (for sampled checks)
    gs_x     optional global scale of x; by default computed from x.  A sampled check passes the
             scale of the whole batch when x holds only some of its rows (a token's output
             depends on the batch only through this scale)

    Returns dict: out float64 (T, H), routing, permutation, gs_x, and (keep=True) per-row
    intermediates c1 (R, 2I), h32 (R, I), h_codes (R, I), h_sf (R, I/16), y (R, H).
    """
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    E = w1.E
    I = w1.N // 2
    if ids is None:
        ids, weights = route_topk(logits, k, renormalize)
    perm = permute(ids, weights, E)
    if gs_x is None:
        gs_x = global_scale(x)
    gs_x = np.float32(gs_x)
    xc, xsf = quantize(x, gs_x)
    out = np.zeros((T, H), dtype=np.float64)
    R = perm["R"]
    inter = {}
    if keep:
        inter = dict(c1=np.zeros((R, 2 * I)), h32=np.zeros((R, I), np.float32),
                     h_codes=np.zeros((R, I), np.uint8), h_sf=np.zeros((R, I // 16), np.uint8),
                     y=np.zeros((R, H)))
    ev = range(E) if experts is None else experts
    for e in ev:
        m = int(perm["counts"][e])
        if m == 0:
            continue
        lo = int(perm["offs"][e])
        rows = np.arange(lo, lo + m)
        tok = perm["row_token"][rows]
        a = dequantize(xc[tok], xsf[tok], gs_x)
        c1 = a @ w1.dequant(e).T
        g, u = c1[:, :I], c1[:, I:]
        h32 = (silu(g) * u).astype(np.float32)
        hc, hsf = quantize(h32, gs_h)
        y = dequantize(hc, hsf, gs_h) @ w2.dequant(e).T
        np.add.at(out, tok, perm["row_w"][rows][:, None] * y)
        if keep:
            inter["c1"][rows] = c1
            inter["h32"][rows] = h32
            inter["h_codes"][rows] = hc
            inter["h_sf"][rows] = hsf
            inter["y"][rows] = y
    res = dict(out=out, ids=ids, weights=weights, perm=perm, gs_x=gs_x, x_codes=xc, x_sf=xsf)
    res.update(inter)
    return res


def bf16_round(v):
    """Round float64 values to bfloat16 (RN-even via float32), returned as float64."""
    f = np.asarray(v, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)
