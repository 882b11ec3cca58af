"""Dense NVFP4 linear and the RMSNorm that feeds the quantizer (oracle side).

Test infrastructure, not product: only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.

What the pages fix
------------------
* A dense NVFP4 linear exists beside the MoE path: the layer ``Nvfp4Linear`` quantizes its
  activation (amax -> gsa on the GPU, then NVFP4 codes against that gsa) and runs an NVFP4
  GEMM against pre-quantized weights; the shared expert does the same for its two projections
  (commit log of dsv4/kernels/cuda, nvfp4-megamoe-kernel: the "Updated layers" list of the
  fused amax + quantize commit).
* An RMSNorm is fused with the quantizer in front of a projection: the fused kernel keeps the
  row's inverse RMS ("s_inv_rms") next to the activation amax (same commit log, the fix of the
  block-reduce scratch that overwrote s_inv_rms).

Readings where the pages are silent
-----------------------------------
* RMSNorm: y = x * (1 / sqrt(mean(x^2) + eps)) * gamma, the standard definition, with this
  FP32 operation order (one rounding per step):
      ss   = sum of x_i^2 over the row, in float64 (each x_i^2 of a bf16 x_i is exact)
      ms   = fl32(ss / cols)                 (float64 quotient, rounded once to float32)
      v    = fl32(ms + eps)
      s    = fl32(sqrt(v))
      rstd = fl32(1 / s)
      y_i  = fl32(fl32(x_i * rstd) * gamma_i)
  The float64 sum is exact for every row whose squares span at most 53 bits, and otherwise
  within one float64 rounding of exact, so any summation order gives the same float32 ms
  except when the exact mean sits within ~1e-16 (relative) of a float32 rounding boundary.
* The quantizer then sees y exactly as it sees any activation: gs = 2688 / max|y| over the
  whole tensor, block scales and codes by :func:`oracle.quant.quantize`.
* Linear: out = dequant(quantize(x)) @ dequant(W)^T in float64, W of shape (N, K) with one
  FP32 global scale; the bf16 output is that value rounded once.
* Shared expert: the expert FFN of the MoE path applied to every token with weight 1 (one
  expert, top-1): [RMSNorm ->] quantize -> L1 -> SwiGLU -> re-quantize with the static gs_h ->
  L2.  It is evaluated by :func:`oracle.moe.moe_ffn` with every token routed to expert 0.
"""

import numpy as np

from .moe import moe_ffn
from .quant import dequantize, global_scale, quantize


def rmsnorm(x, gamma, eps):
    """Row-wise RMSNorm of a (rows, cols) float32 array with weight ``gamma`` (cols,).

    Returns (y float32 (rows, cols), rstd float32 (rows,)), op order as in the module docstring.
    """
    x32 = np.asarray(x, dtype=np.float32)
    g32 = np.asarray(gamma, dtype=np.float32)
    rows, cols = x32.shape
    x64 = x32.astype(np.float64)
    ss = np.sum(x64 * x64, axis=1)                                  # float64 sum of exact squares
    ms = (ss / np.float64(cols)).astype(np.float32)                 # one rounding to float32
    v = (ms + np.float32(eps)).astype(np.float32)
    s = np.sqrt(v).astype(np.float32)                               # IEEE sqrt, correctly rounded
    with np.errstate(divide="ignore"):
        rstd = (np.float32(1.0) / s).astype(np.float32)
    with np.errstate(invalid="ignore", over="ignore"):  # 0 * inf = NaN for an all-zero row, eps 0
        y = (x32 * rstd[:, None]).astype(np.float32)
        y = (y * g32[None, :]).astype(np.float32)
    return y, rstd


def rmsnorm_quantize(x, gamma, eps):
    """RMSNorm, then NVFP4 with the global scale from the amax of the normalized tensor.

    Returns (codes uint8 (rows, cols) unpacked, sf uint8 (rows, cols/16), gs float32, y float32).
    """
    y, _ = rmsnorm(x, gamma, eps)
    gs = global_scale(y)
    codes, sf = quantize(y, gs)
    return codes, sf, gs, y


def linear(x, w_codes, w_sf, gs_w):
    """Dense NVFP4 linear: out (M, N) float64 = dequant(quantize(x)) @ dequant(W)^T.

    ``x`` (M, K) float32 activations (quantized here with gs from their amax); ``w_codes``
    (N, K) unpacked codes, ``w_sf`` (N, K/16) scale bytes, ``gs_w`` the weight's FP32 global
    scale.  Returns (out, dict with the activation's codes, sf and gs).
    """
    x32 = np.asarray(x, dtype=np.float32)
    gs_x = global_scale(x32)
    codes, sf = quantize(x32, gs_x)
    a = dequantize(codes, sf, gs_x)
    b = dequantize(w_codes, w_sf, np.float32(gs_w))
    return a @ b.T, dict(codes=codes, sf=sf, gs=gs_x)


def shared_expert(x, w1, w2, gs_h, gamma=None, eps=1e-6):
    """The shared expert's FFN on every row of x (float32 (M, H)): RMSNorm first when ``gamma``
    is given, then the expert FFN of :func:`oracle.moe.moe_ffn` with one expert (``w1``, ``w2``
    QuantWeights with E = 1) and every token routed to it with weight 1.  Returns float64 (M, H).
    """
    x32 = np.asarray(x, dtype=np.float32)
    if gamma is not None:
        x32, _ = rmsnorm(x32, gamma, eps)
    M = x32.shape[0]
    ids = np.zeros((M, 1), dtype=np.int32)
    w = np.ones((M, 1), dtype=np.float64)
    return moe_ffn(x32, None, 1, w1, w2, np.float32(gs_h), ids=ids, weights=w)["out"]
