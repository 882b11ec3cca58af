"""CPU oracle for the NVFP4 MoE expert-FFN path: test infrastructure, not product.

Plain, slow, float64 numpy restatement of what the path computes, written from the
nvfp4-megamoe-kernel pages and the published FP4/FP8 format definitions.  Only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it;
the library and its Python binding never do, and the oracle imports nothing from them.

Modules
-------
formats   E2M1 / E4M3 codecs and nibble packing
quant     NVFP4 quantizer (global scale from amax, FP8-round-tripped block scale),
          dequantizer, and the 128x4 scale-factor tile index map
routing   softmax top-k routing and the expert-bucketed row permutation
moe       grouped GEMM, SwiGLU, re-quantization, weighted scatter, whole FFN
dense     dense NVFP4 linear, and the RMSNorm fused in front of the quantizer
mx        MXFP4 (32-element blocks, UE8M0 scales), the format the pages contrast with NVFP4

Every function says which page passage it follows.  Functions with no independent pin say
"parity unpinned" in their docstring.
"""

from . import formats, quant, routing, moe, dense, mx  # noqa: F401
