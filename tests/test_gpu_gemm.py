"""GPU parity: the plain 2D x 3D block-scaled grouped GEMM (tcgen05, TMEM accumulation) on
identical quantized operands, against the oracle's float64 grouped GEMM."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import moe as M
from oracle import quant as Q
from tests._gpu_util import DEV, rel_fro, to_dev, upload_nvfp4

pytestmark = pytest.mark.gpu


def _problem(seed, E, N, K, m_sizes):
    """Quantized A (segments padded to 128 rows, padding rows zero) and per-expert B, made by the
    oracle; returns device operands and the oracle's float64 result."""
    rng = np.random.default_rng(seed)
    padded = [(m + 127) // 128 * 128 for m in m_sizes]
    offs = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    Rr = int(offs[-1])
    a = np.zeros((Rr, K), np.float32)
    for e, m in enumerate(m_sizes):
        a[offs[e]:offs[e] + m] = rng.standard_normal((m, K))
    a = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    gs_a = Q.global_scale(a)
    ac, asf = Q.quantize(a, gs_a)
    wf = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    wf = torch.from_numpy(wf).to(torch.bfloat16).float().numpy()
    w = M.QuantWeights.from_float(wf)
    ref = M.grouped_gemm(Q.dequantize(ac, asf, gs_a), w.dequant, offs, rows_valid=m_sizes)
    a_codes, a_sf = upload_nvfp4(ac, asf)
    wd = nv.NVFP4Weights(to_dev(w.codes.reshape(E * N, K // 2)),
                         to_dev(Q.tile_sf(w.sf.reshape(E * N, K // 16))), to_dev(w.gs), E, N, K)
    return a_codes, a_sf, to_dev(np.array([gs_a], np.float32)), wd, to_dev(offs), ref, offs


def _valid_rows(offs, m_sizes):
    return np.concatenate([np.arange(offs[e], offs[e] + m) for e, m in enumerate(m_sizes)])


@pytest.mark.parametrize("K", [64, 192, 256, 320, 1024])
def test_grouped_gemm_fp32_small(K):
    m_sizes = [1, 0, 129, 127]
    a, asf, gs_a, w, offs_d, ref, offs = _problem(K, 4, 256, K, m_sizes)
    out = nv.grouped_gemm(a, asf, gs_a, w, offs_d, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = _valid_rows(offs, m_sizes)
    got = out.cpu().numpy()[rows]
    assert rel_fro(got, ref[rows]) <= 1e-5
    # padding rows of A are zero -> zero output
    pad = np.setdiff1d(np.arange(offs[-1]), rows)
    assert np.all(out.cpu().numpy()[pad] == 0)


def test_grouped_gemm_several_n_tiles_and_bf16_out():
    m_sizes = [300, 5, 128]
    a, asf, gs_a, w, offs_d, ref, offs = _problem(5, 3, 768, 512, m_sizes)
    rows = _valid_rows(offs, m_sizes)
    out32 = nv.grouped_gemm(a, asf, gs_a, w, offs_d, out_dtype=torch.float32)
    out16 = nv.grouped_gemm(a, asf, gs_a, w, offs_d, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert rel_fro(out32.cpu().numpy()[rows], ref[rows]) <= 1e-5
    # the bf16 epilogue rounds the same FP32 values once
    assert torch.equal(out16.cpu(), out32.cpu().to(torch.bfloat16))
    got16 = out16.float().cpu().numpy()[rows]
    assert rel_fro(got16, M.bf16_round(ref[rows])) <= 1e-3


def test_grouped_gemm_full_k_and_n():
    """K = 7168, N = 4096 (the sweep's GEMM shape) on two small groups."""
    m_sizes = [200, 7]
    a, asf, gs_a, w, offs_d, ref, offs = _problem(9, 2, 4096, 7168, m_sizes)
    out = nv.grouped_gemm(a, asf, gs_a, w, offs_d, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = _valid_rows(offs, m_sizes)
    assert rel_fro(out.cpu().numpy()[rows], ref[rows]) <= 1e-5


@pytest.mark.parametrize("m_sizes,K", [([1100, 0, 2200], 320), ([1153, 900], 1024)])
def test_grouped_gemm_pair_tiles(m_sizes, K):
    """Enough rows per group for 256-row tiles on CTA pairs: groups with an odd number of
    128-row blocks (the pair's second half past the group, for the last group past the end of A),
    an empty group, a partial last K stage, two N-tiles."""
    E = len(m_sizes)
    a, asf, gs_a, w, offs_d, ref, offs = _problem(11 + K, E, 512, K, m_sizes)
    assert offs[-1] >= 1024 * E  # the library's pair-tile rule
    out = torch.full((int(offs[-1]), 512), 7.0, dtype=torch.float32, device=DEV)
    nv.grouped_gemm(a, asf, gs_a, w, offs_d, out_dtype=torch.float32, out=out)
    torch.cuda.synchronize()
    rows = _valid_rows(offs, m_sizes)
    got = out.cpu().numpy()
    assert rel_fro(got[rows], ref[rows]) <= 1e-5
    # every row of every segment is written (padding rows of A are zero -> zero output)
    pad = np.setdiff1d(np.arange(offs[-1]), rows)
    assert np.all(got[pad] == 0)


def test_grouped_gemm_rejects_bad_shapes():
    z = torch.zeros(256, dtype=torch.uint8, device=DEV)
    f = torch.ones(4, dtype=torch.float32, device=DEV)
    offs = torch.zeros(3, dtype=torch.int32, device=DEV)
    w = nv.NVFP4Weights(z, z, f, 2, 200, 64)  # N % 256 != 0
    with pytest.raises(nv.Nvfp4Error) as ei:
        nv.grouped_gemm(torch.zeros(128, 32, dtype=torch.uint8, device=DEV), z, f, w, offs)
    assert ei.value.code == 2
