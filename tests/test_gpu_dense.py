"""GPU parity: the fused RMSNorm + quantize (bit-exact codes, scales and global scale), the dense
GEMM on NVFP4 activations and the dense NVFP4 linear, against the oracle."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import dense as D
from oracle import formats as F
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_dense
from tests._gpu_util import DEV, cosine, download_nvfp4, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _inputs(rows, cols, seed, gamma_sd=0.3):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(rows, cols, generator=g) * 2.0).to(torch.bfloat16)
    gamma = (1.0 + gamma_sd * torch.randn(cols, generator=g)).to(torch.bfloat16)
    return x, gamma


def _check_rmsnorm_quantize(x, gamma, eps, gs_given=None, dst=None, k=1, out_rows=None,
                            tokens=None):
    gs_in = None if gs_given is None else torch.tensor([gs_given], dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    codes, sf, gs = nv.rmsnorm_quantize(x.to(DEV), gamma.to(DEV), eps, gs=gs_in, dst_row=dst, k=k,
                                        out_rows=out_rows, status=status)
    torch.cuda.synchronize()
    assert nv.read_status(status) == (0, 0)
    y, _ = D.rmsnorm(x.float().numpy(), gamma.float().numpy(), eps)
    gs_o = Q.global_scale(y) if gs_given is None else np.float32(gs_given)
    assert gs.cpu().numpy()[0].view(np.uint32) == np.float32(gs_o).view(np.uint32)
    c_ref, s_ref = Q.quantize(y, gs_o)
    rows, cols = y.shape
    c, s = download_nvfp4(codes, sf, codes.shape[0], cols)
    if tokens is None:
        assert np.array_equal(c[:rows], c_ref)
        assert np.array_equal(s[:rows], s_ref)
    else:
        valid = tokens >= 0
        assert np.array_equal(c[valid], c_ref[tokens[valid]])
        assert np.array_equal(s[valid], s_ref[tokens[valid]])


@pytest.mark.parametrize("shape", [(1, 64), (37, 192), (129, 256), (300, 7168), (8, 4096)])
@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_rmsnorm_quantize_bit_exact(shape, eps):
    x, gamma = _inputs(*shape, seed=shape[0] * 31 + shape[1])
    _check_rmsnorm_quantize(x, gamma, eps)


def test_rmsnorm_quantize_large_eps_and_tiny_rows():
    # eps dominates rows of tiny values; one all-zero row (eps > 0 keeps rstd finite)
    x, gamma = _inputs(40, 512, seed=3)
    x[5:9] *= 1e-3
    x[20] = 0
    _check_rmsnorm_quantize(x, gamma, 0.5)


def test_rmsnorm_quantize_static_scale():
    x, gamma = _inputs(64, 1024, seed=4)
    _check_rmsnorm_quantize(x, gamma, 1e-5, gs_given=37.5)


def test_rmsnorm_quantize_permuted_write():
    """The MoE form: each normalized token goes straight to its k expert rows."""
    T, H, E, k = 50, 512, 6, 2
    x, gamma = _inputs(T, H, seed=5)
    lg = torch.randn(T, E, generator=torch.Generator().manual_seed(6)).numpy()
    ids, w = R.route_topk(lg, k)
    perm = R.permute(ids, w, E)
    dst = to_dev(perm["dst_row"].reshape(-1).astype(np.int32))
    _check_rmsnorm_quantize(x, gamma, 1e-6, dst=dst, k=k, out_rows=perm["R"],
                            tokens=perm["row_token"])


def _weights(N, K, seed):
    g = torch.Generator().manual_seed(seed)
    wf = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).float().numpy()
    qw = M.QuantWeights.from_float(wf[None])
    dev = nv.NVFP4Weights(to_dev(qw.codes.reshape(N, K // 2)),
                          to_dev(Q.tile_sf(qw.sf.reshape(N, K // 16))), to_dev(qw.gs), 1, N, K)
    return qw, dev


def _assert_close(got, ref):
    """bf16 output against the float64 oracle: one bf16 rounding (half an ulp, at most 2^-8 of
    the value) plus FP32 accumulation noise (about sqrt(K) * 2^-24 of the output's RMS, bounded
    here by 1e-4 of it); and the output-level acceptance bars."""
    got = np.asarray(got, np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * rms
    assert np.all(err <= bound), float(np.max(err - bound))
    assert rel_fro(got, M.bf16_round(ref)) <= 1e-3
    assert cosine(got, ref) >= 0.9999


# (M, N, K): one 128-row tile, ragged rows, split-K (N = 256 leaves most SMs idle), the pair
# tiles from 1024 rows, and the full decode shape of the shared expert's gate/up projection
LINEAR_CASES = [(1, 256, 64), (16, 256, 1024), (100, 768, 1024), (130, 512, 512),
                (1100, 256, 256), (2304, 512, 320), (16, 4096, 7168)]


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("mnk", LINEAR_CASES)
def test_linear_parity(mnk, norm):
    Mr, N, K = mnk
    x, gamma = _inputs(Mr, K, seed=Mr + N + K)
    qw, wd = _weights(N, K, seed=N * 7 + K)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = nv.linear(x.to(DEV), wd, gamma=gamma.to(DEV) if norm else None, eps=1e-6, status=status)
    torch.cuda.synchronize()
    assert nv.read_status(status) == (0, 0)
    xf = x.float().numpy()
    if norm:
        xf, _ = D.rmsnorm(xf, gamma.float().numpy(), 1e-6)
    ref, _ = D.linear(xf, F.unpack_nibbles(qw.codes[0]), qw.sf[0], qw.gs[0])
    _assert_close(out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("mnk", [(16, 4096, 7168), (200, 512, 2048), (1, 768, 64)])
def test_gemm_dense_on_quantized_activations(mnk):
    """nvfp4_gemm_dense on the output of nvfp4_quantize, with garbage in the padding rows."""
    Mr, N, K = mnk
    x, _ = _inputs(Mr, K, seed=9 + Mr)
    qw, wd = _weights(N, K, seed=K)
    Mp = (Mr + 127) // 128 * 128
    codes, sf, gs = nv.quantize(x.to(DEV), out_rows=Mp)
    codes[Mr:] = 0x77  # padding rows: +6 everywhere, never stored
    out = nv.gemm_dense(codes, sf, gs, Mr, wd)
    torch.cuda.synchronize()
    c, s = download_nvfp4(codes, sf, Mp, K)
    a = Q.dequantize(c[:Mr], s[:Mr], float(gs.item()))
    ref = a @ qw.dequant(0).T
    _assert_close(out.float().cpu().numpy(), ref)


def test_linear_reproducible_and_zero_rows():
    x, gamma = _inputs(16, 2048, seed=13)
    _, wd = _weights(1024, 2048, seed=14)
    xd, gd = x.to(DEV), gamma.to(DEV)
    a = nv.linear(xd, wd, gamma=gd)
    b = nv.linear(xd, wd, gamma=gd)
    assert torch.equal(a, b)  # split-K partials are added in a fixed order
    empty = nv.linear(xd[:0], wd)
    assert empty.shape == (0, 1024)


def test_linear_prefill_size_sampled_rows():
    """The dense prefill workload (8192 x 7168 -> 4096, RMSNorm fused) in the launch the bench
    times; sampled rows against the oracle (the whole-tensor amax is exact on the host)."""
    cfg = CONFIGS["dense_prefill"]
    x, gamma, w = gen_dense(cfg)
    qw = M.QuantWeights.from_float(w.float().numpy()[None])
    wd = nv.NVFP4Weights(to_dev(qw.codes.reshape(cfg.N, cfg.K // 2)),
                         to_dev(Q.tile_sf(qw.sf.reshape(cfg.N, cfg.K // 16))), to_dev(qw.gs), 1,
                         cfg.N, cfg.K)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = nv.linear(x.to(DEV), wd, gamma=gamma.to(DEV), eps=cfg.eps, status=status)
    torch.cuda.synchronize()
    assert nv.read_status(status) == (0, 0)
    y, _ = D.rmsnorm(x.float().numpy(), gamma.float().numpy(), cfg.eps)
    gs = Q.global_scale(y)
    rows = np.array([0, 1, 127, 128, 4095, 6000, 8191])
    c, s = Q.quantize(y[rows], gs)
    ref = Q.dequantize(c, s, gs) @ qw.dequant(0).T
    _assert_close(out[torch.from_numpy(rows)].float().cpu().numpy(), ref)


def _expert_weights(H, I, seed, scale=0.02):
    from tests._gpu_util import upload_weights
    g = torch.Generator().manual_seed(seed)
    w1f = (torch.randn(1, 2 * I, H, generator=g) * scale).to(torch.bfloat16).float().numpy()
    w2f = (torch.randn(1, H, I, generator=g) * scale).to(torch.bfloat16).float().numpy()
    q1, q2 = M.QuantWeights.from_float(w1f), M.QuantWeights.from_float(w2f)
    return q1, q2, upload_weights(q1, w1=True), upload_weights(q2)


# (M, H, I, gs_h): one tile, ragged rows, pair tiles from 1024 rows, and the decode shape of the
# model's shared expert (hidden 7168, intermediate 2048; split-K down projection)
SHARED_CASES = [(1, 256, 128, 64.0), (37, 256, 128, 64.0), (200, 512, 256, 64.0),
                (1100, 256, 128, 64.0), (16, 7168, 2048, 1.0)]


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("case", SHARED_CASES)
def test_shared_expert_parity(case, norm):
    Mr, H, I, gs_h = case
    x, gamma = _inputs(Mr, H, seed=Mr * 3 + H)
    q1, q2, w1, w2 = _expert_weights(H, I, seed=H + I)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gs_h_d = torch.tensor([gs_h], dtype=torch.float32, device=DEV)
    out = nv.shared_expert(x.to(DEV), w1, w2, gs_h_d, gamma=gamma.to(DEV) if norm else None,
                           eps=1e-6, status=status)
    torch.cuda.synchronize()
    assert nv.read_status(status) == (0, 0)
    ref = D.shared_expert(x.float().numpy(), q1, q2, np.float32(gs_h),
                          gamma=gamma.float().numpy() if norm else None, eps=1e-6)
    got = out.float().cpu().numpy()
    # the intermediate is re-quantized (a rare one-step E2M1 difference is allowed there), so
    # the bars are the output-level ones of the MoE FFN
    assert rel_fro(got, M.bf16_round(ref)) <= 1e-3
    assert cosine(got, ref) >= 0.9999
