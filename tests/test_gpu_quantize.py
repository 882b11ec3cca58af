"""GPU parity: nvfp4_quantize (amax -> gs on the device, FP8-round-tripped block scale) against
the oracle, bit-exact on codes, scales and the global scale."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_logits, gen_x
from tests._gpu_util import DEV, download_nvfp4, to_dev

pytestmark = pytest.mark.gpu


def _check(x_bf16, gs_given=None, dst=None, k=1, out_rows=None, tokens=None):
    xd = x_bf16.to(DEV)
    gs_in = None if gs_given is None else torch.tensor([gs_given], dtype=torch.float32, device=DEV)
    codes, sf, gs = nv.quantize(xd, gs=gs_in, dst_row=dst, k=k, out_rows=out_rows)
    torch.cuda.synchronize()
    xf = x_bf16.float().numpy()
    gs_o = Q.global_scale(xf) if gs_given is None else np.float32(gs_given)
    assert gs.cpu().numpy()[0].view(np.uint32) == np.float32(gs_o).view(np.uint32)
    c_ref, s_ref = Q.quantize(xf, gs_o)
    rows, cols = xf.shape
    c, s = download_nvfp4(codes, sf, codes.shape[0], cols)
    if tokens is None:
        assert np.array_equal(c[:rows], c_ref)
        assert np.array_equal(s[:rows], s_ref)
    else:  # permuted: row r holds token tokens[r]
        valid = tokens >= 0
        assert np.array_equal(c[valid], c_ref[tokens[valid]])
        assert np.array_equal(s[valid], s_ref[tokens[valid]])


@pytest.mark.parametrize("shape", [(1, 64), (3, 128), (129, 256), (64, 7168), (300, 320)])
def test_quantize_normal(shape):
    g = torch.Generator().manual_seed(shape[0] * 7 + shape[1])
    _check(torch.randn(*shape, generator=g).to(torch.bfloat16))


def test_quantize_outliers_and_tiny_values():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(256, 512, generator=g)
    x[torch.rand(256, 512, generator=g) < 0.01] *= 50
    x[:32] *= 1e-4
    x[40, :16] = 0.0
    x[41, :16] = -0.0
    _check(x.to(torch.bfloat16))


def test_quantize_given_scale_hits_every_tie():
    """With gs = 1 and a block amax of 6, d = 1 and x * r = x: every E2M1 tie point, both
    signs and -0 go straight into the converter."""
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 0.0, 0.125]
    row = np.array([6.0] + vals, dtype=np.float32)
    x = np.stack([row, -row, np.array([6.0] + [-0.0] * 15, np.float32)])
    # E4M3 ties of the block scale: amax = 6 * (1 + (2m+1)/16) sits midway between two scales
    amax_rows = [6 * (1 + (2 * m + 1) / 16) for m in range(8)] + [6 * 2.0 ** -10, 6 * 3 * 2.0 ** -10]
    extra = np.zeros((len(amax_rows), 16), np.float32)
    for i, a in enumerate(amax_rows):
        extra[i, 0] = a
        extra[i, 1:] = np.linspace(-a, a, 15)
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)  # exact
    x = np.concatenate([x, extra])  # (linspace interiors are rounded to bf16; the amax is exact)
    x = np.concatenate([x, np.zeros((x.shape[0], 48), np.float32)], axis=1)  # cols 64
    xt = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(xt.float().numpy()[:, 0], x[:, 0])
    _check(xt, gs_given=1.0)


def test_quantize_zero_scale_blocks_give_zero_codes():
    """Blocks far below the global amax: their E4M3 scale rounds to 0 and every code is +0,
    negative elements included."""
    x = torch.zeros(2, 64)
    x[0, 0] = 1000.0
    x[1, :] = -1e-6 * torch.arange(1, 65)
    _check(x.to(torch.bfloat16))


def test_quantize_extreme_small_amax_no_nan():
    """amax 1e-34 gives a finite gs ~ 2.7e37; a block of subnormals gets the smallest scale
    2^-9, so gs / d overflows to inf: its zero elements stay zero, the others saturate."""
    x = torch.zeros(1, 64)
    x[0, 0] = 1e-34
    x[0, 16] = 4.3e-40
    x[0, 17] = -3e-40
    xb = x.to(torch.bfloat16)
    assert xb.float()[0, 16] > 0  # a bf16 subnormal, not flushed
    gs = Q.global_scale(xb.float().numpy())
    assert np.isfinite(gs) and gs > 1e37
    _check(xb)


def test_quantize_all_zero_matrix_gives_unit_scale():
    _check(torch.zeros(5, 64, dtype=torch.bfloat16))


def test_quantize_strided_rows():
    g = torch.Generator().manual_seed(3)
    big = torch.randn(40, 192, generator=g).to(torch.bfloat16)
    xd = big.to(DEV)[:, :128]
    codes, sf, gs = nv.quantize(xd)
    torch.cuda.synchronize()
    xf = big[:, :128].float().numpy()
    gs_o = Q.global_scale(xf)
    c_ref, s_ref = Q.quantize(xf, gs_o)
    c, s = download_nvfp4(codes, sf, 40, 128)
    assert np.array_equal(c, c_ref) and np.array_equal(s, s_ref)


def test_quantize_permuted_write_tiny():
    cfg = CONFIGS["tiny"]
    x = gen_x(cfg)
    ids, w = R.route_topk(gen_logits(cfg).numpy(), cfg.k)
    p = R.permute(ids, w, cfg.E)
    dst = to_dev(p["dst_row"].reshape(-1).astype(np.int32))
    _check(x, dst=dst, k=cfg.k, out_rows=p["R"], tokens=p["row_token"])


def test_quantize_bad_destination_is_flagged_not_written():
    x = torch.ones(2, 64, dtype=torch.bfloat16, device=DEV)
    dst = torch.tensor([0, 5000, -1, 1], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    nv.quantize(x, dst_row=dst, k=2, out_rows=128, status=status)
    code, rc = nv.read_status(status)
    assert code & 2 and rc == 7
