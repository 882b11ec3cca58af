"""CPU checks of the C ABI: the library builds, loads, exports every entry point the header
declares, and rejects bad arguments on the host before touching the GPU."""

import ctypes
import os
import re

import pytest

from nvfp4_block_scaled_gsa_b200 import build as B
from nvfp4_block_scaled_gsa_b200 import _native as N

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "nvfp4_moe.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return N.lib()


def declared_names():
    text = open(HEADER).read()
    return re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(declared_names())
    for must in ["nvfp4_quantize", "moe_permute", "moe_grouped_gemm_l1_swiglu_q",
                 "moe_grouped_gemm_l2_scatter", "moe_ffn_forward", "nvfp4_grouped_gemm"]:
        assert must in names


def test_every_declared_symbol_is_exported(L):
    names = declared_names()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(N.SIGNATURES), "binding signatures out of sync with the header"


def test_host_only_queries(L):
    assert L.nvfp4_abi_version() == 1
    assert L.nvfp4_quantize_workspace_size() == 256
    assert L.moe_rows_max(16, 256, 8) == 128 + 127 * 128  # 128 slots, at most 128 busy experts
    assert L.moe_rows_max(8192, 256, 8) == 65536 + 127 * 256
    assert L.moe_rows_max(0, 8, 2) == 0
    assert L.moe_rows_max(64, 8, 2) == 128 + 127 * 8 + 8  # rounded up to 128
    big = L.moe_ffn_workspace_size(8192, 7168, 2048, 256, 8)
    R = L.moe_rows_max(8192, 256, 8)
    assert big >= R * (7168 // 2 + 7168 // 16 + 2048 // 2 + 2048 // 16) + 8192 * 7168 * 4
    assert L.moe_ffn_workspace_size(0, 7168, 2048, 256, 8) > 0
    assert L.moe_ffn_workspace_size(-1, 7168, 2048, 256, 8) == 0


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails host validation


@pytest.mark.parametrize("args,code", [
    # rows, cols, ld, dst, k, out_rows, compute_gs
    ((4, 65, 65, None, 1, 4, 1), 2),     # cols % 64
    ((4, 64, 60, None, 1, 4, 1), 1),     # ld < cols
    ((4, 64, 66, None, 1, 4, 1), 2),     # ld % 8
    ((4, 64, 64, None, 1, 2, 1), 1),     # out_rows < rows without a row map
    ((4, 64, 64, FAKE, 0, 4, 1), 1),     # k = 0
    ((-1, 64, 64, None, 1, 4, 1), 1),    # negative rows
])
def test_quantize_rejects_bad_arguments(L, args, code):
    rows, cols, ld, dst, k, out_rows, comp = args
    rc = L.nvfp4_quantize(FAKE, rows, cols, ld, dst, k, out_rows, FAKE, FAKE, FAKE, comp, FAKE,
                          256, None, None)
    assert rc == code


def test_quantize_rejects_misaligned_and_small_workspace(L):
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.nvfp4_quantize(odd, 4, 64, 64, None, 1, 4, FAKE, FAKE, FAKE, 1, FAKE, 256, None,
                            None) == 3
    assert L.nvfp4_quantize(FAKE, 4, 64, 64, None, 1, 4, FAKE, FAKE, FAKE, 1, FAKE, 4, None,
                            None) == 4


def test_permute_rejects_bad_shapes(L):
    f = FAKE
    assert L.moe_permute(f, 4, 0, 1, 1, f, f, f, f, f, f, None, 0, None, None) == 2     # E = 0
    assert L.moe_permute(f, 4, 300, 8, 1, f, f, f, f, f, f, None, 0, None, None) == 2   # E > 256
    assert L.moe_permute(f, 4, 8, 9, 1, f, f, f, f, f, f, None, 0, None, None) == 2     # k > E
    assert L.moe_permute(f, 4, 64, 33, 1, f, f, f, f, f, f, None, 0, None, None) == 2   # k > 32
    assert L.moe_permute(f, 4, 8, 2, 1, f, f, None, f, f, f, None, 0, None, None) == 1  # offs


def test_gemms_reject_bad_shapes(L):
    f = FAKE
    assert L.nvfp4_grouped_gemm(f, f, f, f, f, f, f, 2, 200, 64, 128, f, 0, None, None) == 2
    assert L.nvfp4_grouped_gemm(f, f, f, f, f, f, f, 2, 256, 96, 128, f, 0, None, None) == 2
    assert L.nvfp4_grouped_gemm(f, f, f, f, f, f, f, 2, 256, 64, 100, f, 0, None, None) == 2
    assert L.nvfp4_grouped_gemm(f, f, f, f, f, f, f, 2, 256, 64, 128, f, 7, None, None) == 1
    assert L.moe_grouped_gemm_l1_swiglu_q(f, f, f, f, f, f, f, None, 8, 256, 96, 128, f, f, f,
                                          None, None) == 2  # I % 128
    assert L.moe_grouped_gemm_l2_scatter(f, f, f, f, f, f, f, f, f, f, 8, 200, 128, 4, 2, 128, f,
                                         f, None, None, None) == 2  # H % 128
    assert L.moe_grouped_gemm_l2_scatter(f, f, f, f, f, f, f, f, f, f, 8, 256, 128, 4, 2, 128, f,
                                         None, None, None, None) == 1  # no output
    assert L.moe_grouped_gemm_l2_scatter_noalloc(f, f, f, f, f, f, f, f, f, f, 8, 256, 128, 4096,
                                                 2, 128, f, None, None) == 4  # T*k*H > 1<<20
    assert L.moe_ffn_forward(f, f, 4, 256, 128, 8, 2, f, f, f, f, f, f, f, f, f, 10, None,
                             None) == 4  # workspace too small
    assert L.moe_ffn_forward(f, f, 4, 256, 128, 8, 2, f, f, f, f, f, f, f, f, None, 1 << 30, None,
                             None) == 1


def test_wait_selftest_rejects_bad_arguments(L):
    f = FAKE
    assert L.nvfp4_wait_selftest(0, f, None, None) == 1
    assert L.nvfp4_wait_selftest(3_000_000_000, f, None, None) == 1  # above the 2 s wait limit
    assert L.nvfp4_wait_selftest(10_000_000, None, None, None) == 1


def test_w1_row_map_is_the_documented_interleave(L):
    I = 192
    buf = (ctypes.c_int32 * (2 * I))()
    assert L.moe_w1_row_map(I, ctypes.cast(buf, ctypes.c_void_p)) == 0
    m = list(buf)
    assert sorted(m) == list(range(2 * I))
    for r in (0, 1, 15, 16, 63, 64, 100, 191):
        assert m[r] == 32 * (r // 16) + r % 16            # gate row r
        assert m[I + r] == 32 * (r // 16) + 16 + r % 16   # up row r
    assert m[:3] == [0, 1, 2] and m[16] == 32 and m[I] == 16
    assert L.moe_w1_row_map(100, ctypes.cast(buf, ctypes.c_void_p)) == 1  # I % 16


def test_dense_workspace_sizes(L):
    # amax word + one float per row, in 256-byte units
    assert L.nvfp4_rmsnorm_quantize_workspace_size(8192) == 256 + 8192 * 4
    assert L.nvfp4_rmsnorm_quantize_workspace_size(1) == 512
    assert L.nvfp4_rmsnorm_quantize_workspace_size(0) == 256
    # M = 16, N = 4096, K = 7168: quantizer scratch, gs, 128 padded code rows and their scales,
    # and 9 K ranges of FP32 partials (16 output tiles, 148 // 16 = 9 CTAs per tile)
    want = 512 + 256 + 128 * 3584 + 128 * 448 + 9 * 16 * 4096 * 4
    assert L.nvfp4_linear_workspace_size(16, 4096, 7168) == want
    # 8192 rows give 512 tiles: no split, no partials
    assert L.nvfp4_linear_workspace_size(8192, 4096, 7168) == (
        256 + 8192 * 4 + 256 + 8192 * 3584 + 8192 * 448)
    # K = 256 has one stage: no split either
    assert L.nvfp4_linear_workspace_size(16, 4096, 256) == 512 + 256 + 128 * 128 + 128 * 16
    assert L.nvfp4_linear_workspace_size(-1, 4096, 256) == 0


def test_dense_entry_points_reject_bad_arguments(L):
    f = FAKE
    odd = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 40
    lin = L.nvfp4_linear
    # x, M, K, ld, gamma, eps, w, sfw, gs_w, N, out, ws, ws_bytes, status, stream
    assert lin(f, 16, 100, 128, None, 0.0, f, f, f, 256, f, f, big, None, None) == 2  # K % 64
    assert lin(f, 16, 128, 128, None, 0.0, f, f, f, 200, f, f, big, None, None) == 2  # N % 256
    assert lin(f, 16, 128, 64, None, 0.0, f, f, f, 256, f, f, big, None, None) == 1   # ld < K
    assert lin(f, 16, 128, 128, None, -1.0, f, f, f, 256, f, f, big, None, None) == 1  # eps < 0
    assert lin(f, 16, 128, 128, None, 0.0, f, f, f, 256, f, f, 64, None, None) == 4   # workspace
    assert lin(odd, 16, 128, 128, None, 0.0, f, f, f, 256, f, f, big, None, None) == 3
    assert lin(f, 16, 128, 128, odd, 0.0, f, f, f, 256, f, f, big, None, None) == 3  # gamma
    assert lin(f, 16, 128, 128, None, 0.0, None, f, f, 256, f, f, big, None, None) == 1
    assert lin(None, 0, 128, 128, None, 0.0, f, f, f, 256, None, f, big, None, None) == 0  # M = 0
    rq = L.nvfp4_rmsnorm_quantize
    # x, rows, cols, ld, gamma, eps, dst, k, out_rows, codes, sf, gs, compute, ws, ws_bytes, ...
    assert rq(f, 4, 64, 64, f, float("nan"), None, 1, 4, f, f, f, 1, f, big, None, None) == 1
    assert rq(f, 4, 64, 64, None, 0.0, None, 1, 4, f, f, f, 1, f, big, None, None) == 1  # gamma
    assert rq(f, 4, 64, 64, f, 0.0, None, 1, 4, f, f, f, 1, f, 256, None, None) == 4   # ws
    assert rq(f, 4, 96, 96, f, 0.0, None, 1, 4, f, f, f, 1, f, big, None, None) == 2   # cols % 64
    assert rq(f, 4, 64, 64, odd, 0.0, None, 1, 4, f, f, f, 1, f, big, None, None) == 3


def test_shared_expert_workspace_and_argument_checks(L):
    # quantizer scratch, gs, x codes + scales, h codes + scales (128 padded rows each), 5 K
    # ranges of FP32 partials for the down projection (28 output tiles: 148 // 28 = 5) and 9 for
    # the L1 (16 output tiles of 2I = 4096 columns: 148 // 16 = 9)
    want = (512 + 256 + 128 * 3584 + 128 * 448 + 128 * 1024 + 128 * 128 + 5 * 16 * 7168 * 4
            + 9 * 16 * 4096 * 4)
    assert L.nvfp4_shared_expert_workspace_size(16, 7168, 2048) == want
    assert L.nvfp4_shared_expert_workspace_size(-1, 7168, 2048) == 0
    # 8192 rows: no split anywhere (fused-epilogue L1, direct bf16 down projection)
    assert L.nvfp4_shared_expert_workspace_size(8192, 7168, 2048) == (
        256 + 8192 * 4 + 256 + 8192 * 3584 + 8192 * 448 + 8192 * 1024 + 8192 * 128)
    f = FAKE
    big = 1 << 40
    se = L.nvfp4_shared_expert
    # x, M, H, ld, gamma, eps, w1, sfw1, gs_w1, w2, sfw2, gs_w2, I, gs_h, out, ws, ws_bytes, ...
    assert se(f, 16, 200, 200, None, 0.0, f, f, f, f, f, f, 128, f, f, f, big, None, None) == 2
    assert se(f, 16, 256, 256, None, 0.0, f, f, f, f, f, f, 64, f, f, f, big, None, None) == 2
    assert se(f, 16, 256, 128, None, 0.0, f, f, f, f, f, f, 128, f, f, f, big, None, None) == 1
    assert se(f, 16, 256, 256, None, 0.0, f, f, f, f, f, f, 128, None, f, f, big, None,
              None) == 1  # no gs_h
    assert se(f, 16, 256, 256, None, 0.0, f, f, f, f, f, f, 128, f, f, f, 100, None, None) == 4
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert se(f, 16, 256, 256, None, 0.0, f, f, f, odd, f, f, 128, f, f, f, big, None, None) == 3
    assert se(None, 0, 256, 256, None, 0.0, f, f, f, f, f, f, 128, f, None, f, big, None,
              None) == 0
