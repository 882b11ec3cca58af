"""GPU parity of the MXFP4 path (E2M1 elements, UE8M0 scale per 32, no global scale) against the
oracle's MXFP4 (oracle/mx.py, the OCP Microscaling rule): codes and scale bytes bit-exact."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from oracle import formats as F
from oracle import mx as X
from oracle import quant as Q
from tests._gpu_util import DEV

pytestmark = pytest.mark.gpu


def _bf16_blocks(rows, cols, seed):
    """bf16 values whose 32-element blocks span magnitudes 2^-140 .. 2^120, with all-zero blocks,
    single-element blocks, blocks whose amax sits on a power of two, and E2M1 midpoints."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    nb = cols // 32
    mag = torch.exp2(torch.randint(-140, 121, (rows, nb), generator=g).float())
    x = (x.view(rows, nb, 32) * mag[..., None]).view(rows, cols)
    special = [
        torch.zeros(32),                                                  # all-zero block
        torch.tensor([0.0] * 8 + [-3.0] + [0.0] * 23),                    # one element
        torch.tensor([4.0] + [0.125 * i for i in range(31)]),            # amax on 2^2
        torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4),  # E2M1 midpoints
        torch.tensor([7.5, -7.0, 6.5, 0.3] * 8),                          # saturating at 6
    ]
    for i, blk in enumerate(special):
        r, c = divmod(i, nb)
        if r < rows:
            x[r, 32 * c:32 * c + 32] = blk
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(1, 128), (130, 256), (257, 7168), (64, 2048)])
def test_mxfp4_quantize_bit_exact(rows, cols):
    x = _bf16_blocks(rows, cols, seed=rows + cols)
    codes, sf = nv.mxfp4_quantize(x.to(DEV))
    torch.cuda.synchronize()
    want_c, want_s = X.quantize_mxfp4(x.float().numpy())
    got_c = F.unpack_nibbles(codes.cpu().numpy())
    got_s = Q.untile_sf(sf.cpu().numpy(), (rows + 127) // 128 * 128, cols // 32)[:rows]
    assert np.array_equal(got_s, want_s)
    # +-0 decode alike: compare the codes of nonzero values bit-exactly, zeros by magnitude
    nz = (want_c & 7) != 0
    assert np.array_equal(got_c[nz], want_c[nz])
    assert np.all((got_c[~nz] & 7) == 0)


def _mx_operand(x):
    """Oracle MXFP4 of float rows -> (dequantized float64, device codes, device tiled scales)."""
    c, sc = X.quantize_mxfp4(x)
    rows, cols = x.shape
    r128 = (rows + 127) // 128 * 128
    cp = np.zeros((r128, cols), np.uint8)
    cp[:rows] = c
    sp = np.zeros((r128, cols // 32), np.uint8)
    sp[:rows] = sc
    return (X.dequantize_mxfp4(c, sc), torch.from_numpy(F.pack_nibbles(cp)).to(DEV),
            torch.from_numpy(Q.tile_sf(sp)).to(DEV))


@pytest.mark.parametrize("E,N,K,rows", [
    (3, 256, 256, [5, 0, 130]),        # ragged segments, an empty expert
    (2, 512, 384, [128, 77]),          # K = 3 * 128: a last stage of two MMAs and one atom
    (2, 4096, 7168, [40, 200]),        # the MoE L1 shape
    (1, 256, 1024, [1100]),            # 9 blocks of 128 rows: 256-row tiles on CTA pairs
])
def test_mxfp4_grouped_gemm_matches_oracle(E, N, K, rows):
    """C = A_e B_e^T on identical MXFP4 operands (the oracle's codes and scales uploaded): FP32
    result within relative Frobenius 1e-5 of the float64 product of the dequantized operands."""
    g = torch.Generator().manual_seed(E * 1000 + K)
    pad = [(m + 127) // 128 * 128 for m in rows]
    offs = np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)
    R = int(offs[-1])
    a = np.zeros((R, K), np.float32)
    for e in range(E):
        a[offs[e]:offs[e] + rows[e]] = (torch.randn(rows[e], K, generator=g) *
                                        torch.exp2(torch.randint(-6, 7, (rows[e], 1),
                                                                 generator=g).float())).numpy()
    b = (torch.randn(E * N, K, generator=g) * 0.02).numpy()
    ad, ac, asf = _mx_operand(a)
    bd, bc, bsf = _mx_operand(b)
    out = nv.mxfp4_grouped_gemm(ac, asf, bc, bsf, E, N, torch.from_numpy(offs).to(DEV))
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for e in range(E):
        lo, hi = offs[e], offs[e] + rows[e]
        if hi == lo:
            continue
        want = ad[lo:hi] @ bd[e * N:(e + 1) * N].T
        err = np.linalg.norm(got[lo:hi] - want) / np.linalg.norm(want)
        assert err <= 1e-5, (e, err)
