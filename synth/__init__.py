"""Seeded synthetic inputs shared by the CUDA-path tests, the oracle checks and the bench.

This package draws random numbers and nothing else: no quantization, routing or GEMM
arithmetic lives here, so both sides of a parity check receive the same inputs without
sharing any of the method's code.
"""

from .inputs import CONFIGS, DenseConfig, MoEConfig, SharedConfig, SweepConfig, gen_dense, gen_logits, gen_shared, gen_x, gen_weight_expert, gen_sweep  # noqa: F401
