"""The bench's algorithmic byte and FLOP counts against hand-written sums (CPU only): every
roofline fraction it reports divides by these."""

import bench
from synth import CONFIGS

B = 0.5 + 1.0 / 16.0  # NVFP4 bytes per element: E2M1 code + one E4M3 scale per 16


def test_moe_step_accounting_decode():
    cfg = CONFIGS["decode"]
    counts = [0] * cfg.E
    for e in range(97):          # 97 active experts with 128 slots between them
        counts[e] = 1
    counts[0] += 128 - 97
    acc = bench.algorithmic(cfg, counts)
    T, H, I, E = 16, 7168, 2048, 256
    w = 97 * 3 * I * H * B
    assert acc["active"] == 97 and acc["slots"] == 128
    assert acc["flops"] == 2 * 128 * (H * 2 * I + I * H)
    assert abs(acc["bytes"] - (w + T * H * 2 + 2 * T * H * B + 2 * 128 * I * B + T * H * 2
                               + T * E * 4)) < 1
    assert abs(acc["l1_bytes"] - (97 * 2 * I * H * B + 128 * H * B + 128 * I * B)) < 1
    assert acc["l1_flops"] == 2 * 128 * H * 2 * I


def test_dense_accounting():
    cfg = CONFIGS["dense_decode"]
    acc = bench.dense_algorithmic(cfg)
    M, N, K = 16, 4096, 7168
    assert acc["flops"] == 2 * M * N * K
    assert abs(acc["gemm_bytes"] - (N * K * B + M * K * B + M * N * 2)) < 1
    assert abs(acc["bytes"] - (M * K * 2 + K * 2 + 2 * M * K * B + N * K * B + M * N * 2)) < 1


def test_shared_accounting():
    cfg = CONFIGS["shared_prefill"]
    acc = bench.shared_algorithmic(cfg)
    M, H, I = 8192, 7168, 2048
    assert acc["flops"] == 6 * M * H * I
    assert acc["l1_flops"] == 4 * M * H * I
    assert abs(acc["l1_bytes"] - (M * H * B + 2 * I * H * B + M * I * B)) < 1
    assert abs(acc["bytes"] - (M * H * 2 + H * 2 + 2 * M * H * B + 3 * I * H * B + 2 * M * I * B
                               + M * H * 2)) < 1


def test_roofline_bound_choice_follows_the_ridge():
    """Decode's L1 (weights streamed for 128 slots) sits far below the FP4 ridge, prefill's
    just below it, the dense prefill GEMM and the shared prefill L1 above it."""
    peaks = dict(hbm=6545.0, bf16=1630.0)
    ridge = peaks["bf16"] * bench.FP4_PER_BF16 * 1e12 / (peaks["hbm"] * 1e9)
    dec = bench.algorithmic(CONFIGS["decode"], [1] * 128 + [0] * 128)
    pre = bench.algorithmic(CONFIGS["prefill"], [256] * 256)
    assert dec["l1_flops"] / dec["l1_bytes"] < ridge
    assert 0.8 * ridge < pre["l1_flops"] / pre["l1_bytes"] < ridge
    dp = bench.dense_algorithmic(CONFIGS["dense_prefill"])
    sp = bench.shared_algorithmic(CONFIGS["shared_prefill"])
    assert dp["flops"] / dp["gemm_bytes"] > ridge
    assert sp["l1_flops"] / sp["l1_bytes"] > ridge


def test_moe_step_kernel_count():
    """The launches the bench line claims per step match the path's kernels: one routing kernel
    below 4096 slots (decode: 128), three from 4096 (mid, prefill), then amax, quantize, L1, L2
    and the combine or bf16 rounding."""
    import nvfp4_block_scaled_gsa_b200 as nv
    assert bench.kernels_per_step(nv, CONFIGS["decode"]) == 6
    assert bench.kernels_per_step(nv, CONFIGS["mid"]) == 8
    assert bench.kernels_per_step(nv, CONFIGS["prefill"]) == 8
