"""Helpers shared by the GPU parity tests: oracle operands -> device buffers, comparisons."""

import numpy as np
import torch

from oracle import formats as F
from oracle import quant as Q

DEV = "cuda"


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(DEV)


def upload_nvfp4(codes_unpacked, sf_logical):
    """Oracle NVFP4 (unpacked codes (R, K), logical scales (R, K/16)) -> device (packed, tiled).
    R must be a multiple of 128."""
    packed = F.pack_nibbles(codes_unpacked)
    tiled = Q.tile_sf(sf_logical)
    return to_dev(packed), to_dev(tiled)


def download_nvfp4(codes_dev, sf_dev, rows, cols):
    """Device (packed codes, tiled scales) -> (unpacked codes (rows, cols), logical scales)."""
    c = F.unpack_nibbles(codes_dev.cpu().numpy())[:rows]
    r128 = (codes_dev.shape[0] + 127) // 128 * 128
    s = Q.untile_sf(sf_dev.cpu().numpy(), r128, cols // 16)[:rows]
    return c, s


def rel_fro(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def cosine(got, want):
    a = np.asarray(got, dtype=np.float64).ravel()
    b = np.asarray(want, dtype=np.float64).ravel()
    return float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))


def e2m1_step(val_abs):
    """Spacing of the E2M1 grid around magnitude val_abs (0.5 below 2, 1 below 4, else 2)."""
    return np.where(val_abs < 2, 0.5, np.where(val_abs < 4, 1.0, 2.0))


def compare_requant(c_gpu, s_gpu, c_ref, s_ref, gs):
    """Re-quantized intermediate: returns (mismatch fraction, count of elements off by more than
    one E2M1 step after dequantization).  A block whose scale byte differs counts all its
    elements as mismatched."""
    rows, cols = c_ref.shape
    scale_diff = np.repeat(s_gpu != s_ref, 16, axis=1)
    mism = (c_gpu != c_ref) | scale_diff
    d_gpu = Q.dequantize(c_gpu, s_gpu, gs)
    d_ref = Q.dequantize(c_ref, s_ref, gs)
    d = np.repeat(F.e4m3_decode(s_ref), 16, axis=1) / np.float64(gs)
    mag = np.abs(F.e2m1_decode(c_ref))
    step = np.maximum(e2m1_step(mag), e2m1_step(np.abs(F.e2m1_decode(c_gpu)))) * d
    far = np.abs(d_gpu - d_ref) > step * (1 + 1e-9) + 1e-30
    return float(mism.mean()), int(far.sum())


def upload_weights(qw, w1=False):
    """Oracle QuantWeights -> device NVFP4Weights.  With w1=True the rows are stored in the
    kernels' gate/up interleave of 16-row blocks (moe_w1_row_map)."""
    import nvfp4_block_scaled_gsa_b200 as nv
    E, N, K2 = qw.codes.shape
    K = 2 * K2
    codes, sf = qw.codes, qw.sf
    if w1:
        m = nv.w1_row_map(N // 2).numpy()
        codes = np.empty_like(qw.codes)
        sf = np.empty_like(qw.sf)
        codes[:, m] = qw.codes
        sf[:, m] = qw.sf
    return nv.NVFP4Weights(to_dev(codes.reshape(E * N, K // 2)),
                           to_dev(Q.tile_sf(sf.reshape(E * N, K // 16))), to_dev(qw.gs), E, N, K)
