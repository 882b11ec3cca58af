"""Torch-facing wrappers over the C ABI: allocate outputs with torch, pass pointers and the
current CUDA stream, check the status.  No arithmetic of the method happens here.
"""

from dataclasses import dataclass

import torch

from ._native import call, lib

U8, I32, F32, BF16 = torch.uint8, torch.int32, torch.float32, torch.bfloat16


def _p(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def round_up(v, m):
    return (v + m - 1) // m * m


def sf_bytes(rows, cols):
    """Bytes of a tiled block-scale buffer for `rows` rows of `cols` elements."""
    return round_up(rows, 128) * cols // 16


@dataclass
class NVFP4Weights:
    """Expert weights (E, N, K) as one NVFP4 tensor of E*N rows: codes (E*N, K/2) uint8, tiled
    scales, global scale per expert (E,) float32."""
    codes: torch.Tensor
    sf: torch.Tensor
    gs: torch.Tensor
    E: int
    N: int
    K: int


def quantize(x, gs=None, dst_row=None, k=1, out_rows=None, status=None):
    """NVFP4-quantize bf16 x (rows, cols).  gs=None: the global scale is computed on the GPU from
    amax (returned as a device tensor); otherwise gs (device float[1]) is used as given.
    dst_row/k/out_rows: permuted write (see nvfp4_quantize in the header)."""
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out_rows is None:
        out_rows = rows
    dev = x.device
    codes = torch.empty(out_rows, cols // 2, dtype=U8, device=dev)
    sf = torch.empty(sf_bytes(out_rows, cols), dtype=U8, device=dev)
    compute = gs is None
    if compute:
        gs = torch.empty(1, dtype=F32, device=dev)
    ws = torch.empty(int(lib().nvfp4_quantize_workspace_size()), dtype=U8, device=dev)
    call("nvfp4_quantize", _p(x), rows, cols, x.stride(0), _p(dst_row), k, out_rows, _p(codes),
         _p(sf), _p(gs), int(compute), _p(ws), ws.numel(), _p(status), _stream())
    return codes, sf, gs


def mxfp4_quantize(x, status=None):
    """MXFP4-quantize bf16 x (rows, cols): returns (codes (rows, cols/2) uint8, tiled UE8M0
    scales, one per 32 elements).  cols % 128 == 0; no global scale."""
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    codes = torch.empty(rows, cols // 2, dtype=U8, device=x.device)
    sf = torch.empty(round_up(rows, 128) * cols // 32, dtype=U8, device=x.device)
    call("mxfp4_quantize", _p(x), rows, cols, x.stride(0), _p(codes), _p(sf), _p(status),
         _stream())
    return codes, sf


def rmsnorm_quantize(x, gamma, eps, gs=None, dst_row=None, k=1, out_rows=None, status=None):
    """RMSNorm of bf16 x (rows, cols) with bf16 gamma (cols,), fused into the NVFP4 quantizer.
    Same outputs and options as quantize(); the normalized tensor itself is never written."""
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1
    assert gamma.dtype == BF16 and gamma.is_contiguous() and gamma.numel() == x.shape[1]
    rows, cols = x.shape
    if out_rows is None:
        out_rows = rows
    dev = x.device
    codes = torch.empty(out_rows, cols // 2, dtype=U8, device=dev)
    sf = torch.empty(sf_bytes(out_rows, cols), dtype=U8, device=dev)
    compute = gs is None
    if compute:
        gs = torch.empty(1, dtype=F32, device=dev)
    ws = torch.empty(int(lib().nvfp4_rmsnorm_quantize_workspace_size(rows)), dtype=U8, device=dev)
    call("nvfp4_rmsnorm_quantize", _p(x), rows, cols, x.stride(0), _p(gamma), float(eps),
         _p(dst_row), k, out_rows, _p(codes), _p(sf), _p(gs), int(compute), _p(ws), ws.numel(),
         _p(status), _stream())
    return codes, sf, gs


def gemm_dense(a_codes, a_sf, gs_a, M, w: "NVFP4Weights", out=None, ws=None, status=None):
    """Dense GEMM on NVFP4 activations (round_up(M, 128) rows of codes and tiled scales):
    bf16 (M, N) = A W^T with W one NVFP4 matrix (w.E == 1)."""
    assert w.E == 1
    if out is None:
        out = torch.empty(M, w.N, dtype=BF16, device=a_codes.device)
    need = int(lib().nvfp4_gemm_dense_workspace_size(M, w.N, w.K))
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=U8, device=a_codes.device)
    call("nvfp4_gemm_dense", _p(a_codes), _p(a_sf), _p(gs_a), M, _p(w.codes), _p(w.sf), _p(w.gs),
         w.N, w.K, _p(out), _p(ws), 0 if ws is None else ws.numel(), _p(status), _stream())
    return out


def linear_workspace_bytes(M, N, K):
    return int(lib().nvfp4_linear_workspace_size(M, N, K))


def linear(x, w: "NVFP4Weights", gamma=None, eps=1e-6, out=None, ws=None, status=None):
    """Dense NVFP4 linear: bf16 x (M, K) -> bf16 (M, N) = x W^T, with W one NVFP4 matrix
    (w.E == 1, shape N x K).  gamma (bf16 (K,)) fuses an RMSNorm into the activation quantizer."""
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1 and w.E == 1
    M, K = x.shape
    assert K == w.K
    if out is None:
        out = torch.empty(M, w.N, dtype=BF16, device=x.device)
    if ws is None:
        ws = torch.empty(max(linear_workspace_bytes(M, w.N, K), 256), dtype=U8, device=x.device)
    call("nvfp4_linear", _p(x), M, K, x.stride(0), _p(gamma), float(eps), _p(w.codes), _p(w.sf),
         _p(w.gs), w.N, _p(out), _p(ws), ws.numel(), _p(status), _stream())
    return out


def shared_expert_workspace_bytes(M, H, I):
    return int(lib().nvfp4_shared_expert_workspace_size(M, H, I))


def shared_expert(x, w1: "NVFP4Weights", w2: "NVFP4Weights", gs_h, gamma=None, eps=1e-6,
                  out=None, ws=None, status=None):
    """The shared expert's FFN on every row of bf16 x (M, H): w1 from quantize_w1 with E = 1
    (gate/up interleave), w2 from quantize_weights with E = 1 (H x I); gs_h device float[1].
    gamma (bf16 (H,)) fuses an RMSNorm into the first quantizer.  Returns bf16 (M, H)."""
    assert x.dtype == BF16 and x.dim() == 2 and x.stride(1) == 1 and w1.E == 1 and w2.E == 1
    M, H = x.shape
    I = w1.N // 2
    assert w1.K == H and w2.N == H and w2.K == I
    if out is None:
        out = torch.empty(M, H, dtype=BF16, device=x.device)
    if ws is None:
        ws = torch.empty(max(shared_expert_workspace_bytes(M, H, I), 256), dtype=U8,
                         device=x.device)
    call("nvfp4_shared_expert", _p(x), M, H, x.stride(0), _p(gamma), float(eps), _p(w1.codes),
         _p(w1.sf), _p(w1.gs), _p(w2.codes), _p(w2.sf), _p(w2.gs), I, _p(gs_h), _p(out), _p(ws),
         ws.numel(), _p(status), _stream())
    return out


def quantize_weights(get_expert, E, N, K, device="cuda", row_map=None):
    """Pre-pack expert weights: get_expert(e) -> bf16 (N, K) on the device; each expert gets its
    own global scale from its amax.  row_map (device int32 [N]): stored row of each row."""
    codes = torch.empty(E * N, K // 2, dtype=U8, device=device)
    sf = torch.empty(E * N * K // 16, dtype=U8, device=device)
    gs = torch.empty(E, dtype=F32, device=device)
    ws = torch.empty(int(lib().nvfp4_quantize_workspace_size()), dtype=U8, device=device)
    per_sf = N * K // 16
    for e in range(E):
        w = get_expert(e)
        assert w.dtype == BF16 and tuple(w.shape) == (N, K)
        w = w.contiguous()
        call("nvfp4_quantize", _p(w), N, K, K, _p(row_map), 1, N, _p(codes[e * N:(e + 1) * N]),
             sf.data_ptr() + e * per_sf, gs.data_ptr() + 4 * e, 1, _p(ws), ws.numel(), None,
             _stream())
    return NVFP4Weights(codes, sf, gs, E, N, K)


def w1_row_map(I):
    """Host int32 [2I]: stored row of each logical W1 row (gate rows, then up rows)."""
    m = torch.empty(2 * I, dtype=I32)
    call("moe_w1_row_map", I, m.data_ptr())
    return m


def quantize_w1(get_expert, E, I, H, device="cuda"):
    """Pre-pack W1 (E experts of [2I][H]: gate rows then up rows) into the kernels' gate/up
    interleave of 16-row blocks (stored row 32j + i = gate row 16j + i, 32j + 16 + i = up row
    16j + i; moe_w1_row_map)."""
    row_map = w1_row_map(I).to(device)
    return quantize_weights(get_expert, E, 2 * I, H, device=device, row_map=row_map)


def rows_max(T, E, k):
    return int(lib().moe_rows_max(T, E, k))


def permute(logits, k, renormalize=True, ids=None, weights=None, E=None, status=None):
    """Top-k routing + expert-bucketed row map.  With logits=None, ids/weights (T, k) are the
    routing (ids < 0 dropped) and E must be given."""
    if logits is not None:
        T, E = logits.shape
        dev = logits.device
        ids = torch.empty(T, k, dtype=I32, device=dev)
        weights = torch.empty(T, k, dtype=F32, device=dev)
    else:
        T = ids.shape[0]
        dev = ids.device
    R = rows_max(T, E, k)
    offs = torch.empty(E + 1, dtype=I32, device=dev)
    dst_row = torch.empty(T * k, dtype=I32, device=dev)
    row_slot = torch.empty(max(R, 1), dtype=I32, device=dev)
    row_w = torch.empty(max(R, 1), dtype=F32, device=dev)
    ws_bytes = lib().moe_permute_workspace_size(T, E, k)
    ws = torch.empty(max(ws_bytes, 1), dtype=U8, device=dev)
    call("moe_permute", _p(logits), T, E, k, int(renormalize), _p(ids), _p(weights), _p(offs),
         _p(dst_row), _p(row_slot), _p(row_w), _p(ws), ws_bytes, _p(status), _stream())
    return dict(ids=ids, weights=weights, offs=offs, dst_row=dst_row, row_slot=row_slot,
                row_w=row_w, R_max=R, E=E, T=T, k=k)


def grouped_gemm(a_codes, a_sf, gs_a, w: NVFP4Weights, offs, out_dtype=F32, status=None,
                 out=None):
    """Plain 2D x 3D grouped GEMM: out[r] = A[r] . W_e^T / (gs_a * gs_w[e]).  Rows past
    offs[E] are left as they are (``out`` may be given, (R, N) of ``out_dtype``)."""
    R = a_codes.shape[0]
    if out is None:
        out = torch.empty(R, w.N, dtype=out_dtype, device=a_codes.device)
    assert out.shape == (R, w.N) and out.dtype == out_dtype and out.is_contiguous()
    call("nvfp4_grouped_gemm", _p(a_codes), _p(a_sf), _p(gs_a), _p(w.codes), _p(w.sf), _p(w.gs),
         _p(offs), w.E, w.N, w.K, R, _p(out), 0 if out_dtype == F32 else 1, _p(status), _stream())
    return out


def mxfp4_grouped_gemm(a_codes, a_sf, b_codes, b_sf, E, N, offs, out_dtype=F32, status=None,
                       out=None):
    """2D x 3D grouped GEMM on MXFP4 operands (mxfp4_quantize's format, no global scales):
    out[r] = A[r] . B_e^T for the rows r of expert e; B is [E*N][K]."""
    R = a_codes.shape[0]
    K = 2 * a_codes.shape[1]
    if out is None:
        out = torch.empty(R, N, dtype=out_dtype, device=a_codes.device)
    assert out.shape == (R, N) and out.dtype == out_dtype and out.is_contiguous()
    call("mxfp4_grouped_gemm", _p(a_codes), _p(a_sf), _p(b_codes), _p(b_sf), _p(offs), E, N, K, R,
         _p(out), 0 if out_dtype == F32 else 1, _p(status), _stream())
    return out


def l1_swiglu_q(a_codes, a_sf, gs_a, w1: NVFP4Weights, offs, gs_h, row_slot=None, status=None):
    """L1 GEMM + SwiGLU + NVFP4 re-quantization -> (h codes (R, I/2), h tiled scales).
    With row_slot, all-padding groups of 32 rows are skipped (left unwritten)."""
    R = a_codes.shape[0]
    I = w1.N // 2
    h = torch.empty(R, I // 2, dtype=U8, device=a_codes.device)
    sfh = torch.empty(sf_bytes(R, I), dtype=U8, device=a_codes.device)
    call("moe_grouped_gemm_l1_swiglu_q", _p(a_codes), _p(a_sf), _p(gs_a), _p(w1.codes),
         _p(w1.sf), _p(w1.gs), _p(offs), _p(row_slot), w1.E, w1.K, I, R, _p(gs_h), _p(h),
         _p(sfh), _p(status), _stream())
    return h, sfh


def l1_swiglu_q_stats(a_codes, a_sf, gs_a, w1: NVFP4Weights, offs, gs_h, row_slot=None,
                      h_stats=None, want_h32=False, status=None):
    """l1_swiglu_q, plus the epilogue's view of h: returns (h codes, h tiled scales, h_stats,
    h32).  h_stats: device uint32 (3,) accumulated into (zeroed here when not given): amax bits
    of |h| over real rows, saturated block scales, underflowed block scales.  h32 (with
    want_h32): the FP32 h values before quantization, (R, I), real rows only."""
    R = a_codes.shape[0]
    I = w1.N // 2
    dev = a_codes.device
    h = torch.empty(R, I // 2, dtype=U8, device=dev)
    sfh = torch.empty(sf_bytes(R, I), dtype=U8, device=dev)
    if h_stats is None:
        h_stats = torch.zeros(3, dtype=I32, device=dev)
    h32 = torch.zeros(R, I, dtype=F32, device=dev) if want_h32 else None
    call("moe_grouped_gemm_l1_swiglu_q_stats", _p(a_codes), _p(a_sf), _p(gs_a), _p(w1.codes),
         _p(w1.sf), _p(w1.gs), _p(offs), _p(row_slot), w1.E, w1.K, I, R, _p(gs_h), _p(h),
         _p(sfh), _p(h32), _p(h_stats), _p(status), _stream())
    return h, sfh, h_stats, h32


def scale_from_amax(amax_bits, gs):
    """gs (device float[1]) = 2688 / amax for the float bits in amax_bits (device 4-byte word),
    1.0 when not finite and positive; on the device, no host sync."""
    call("nvfp4_scale_from_amax", _p(amax_bits), _p(gs), _stream())
    return gs


def l2_scatter(h, sfh, gs_h, w2: NVFP4Weights, offs, row_slot, row_w, dst_row, T, k, status=None):
    """L2 GEMM + routing weight + scatter to token order -> (out fp32 (T, H), out bf16 (T, H))."""
    R = h.shape[0]
    H = w2.N
    I = w2.K
    ys = torch.empty(max(T * k, 1), H, dtype=F32, device=h.device)
    out32 = torch.empty(T, H, dtype=F32, device=h.device)
    out16 = torch.empty(T, H, dtype=BF16, device=h.device)
    call("moe_grouped_gemm_l2_scatter", _p(h), _p(sfh), _p(gs_h), _p(w2.codes), _p(w2.sf),
         _p(w2.gs), _p(offs), _p(row_slot), _p(row_w), _p(dst_row), w2.E, H, I, T, k, R, _p(ys),
         _p(out32), _p(out16), _p(status), _stream())
    return out32, out16


def l2_scatter_add(h, sfh, gs_h, w2: NVFP4Weights, offs, row_slot, row_w, dst_row, T, k,
                   status=None):
    """L2 GEMM + routing weight + scatter-ADD into token rows (reductions at L2, order not fixed)
    -> (out fp32 (T, H), out bf16 (T, H))."""
    R = h.shape[0]
    H, I = w2.N, w2.K
    acc = torch.empty(T, H, dtype=F32, device=h.device)
    out16 = torch.empty(T, H, dtype=BF16, device=h.device)
    call("moe_grouped_gemm_l2_scatter_add", _p(h), _p(sfh), _p(gs_h), _p(w2.codes), _p(w2.sf),
         _p(w2.gs), _p(offs), _p(row_slot), _p(row_w), _p(dst_row), w2.E, H, I, T, k, R,
         _p(acc), _p(out16), _p(status), _stream())
    return acc, out16


def l2_form(T, k, E, deterministic=False):
    """1 when moe_ffn_forward adds L2 rows into token rows for this batch, 0 for slot rows."""
    return int(lib().moe_ffn_l2_form(T, k, E, 2 if deterministic else 0))


def ffn_workspace_bytes(T, H, I, E, k):
    return int(lib().moe_ffn_workspace_size(T, H, I, E, k))


def moe_ffn_forward(x, logits, k, w1: NVFP4Weights, w2: NVFP4Weights, gs_h, out=None, ws=None,
                    status=None):
    """The whole expert FFN: bf16 x (T, H), float logits (T, E) -> bf16 out (T, H)."""
    T, H = x.shape
    E = logits.shape[1]
    I = w1.N // 2
    if out is None:
        out = torch.empty(T, H, dtype=BF16, device=x.device)
    need = ffn_workspace_bytes(T, H, I, E, k)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=U8, device=x.device)
    call("moe_ffn_forward", _p(x), _p(logits), T, H, I, E, k, _p(w1.codes), _p(w1.sf), _p(w1.gs),
         _p(w2.codes), _p(w2.sf), _p(w2.gs), _p(gs_h), _p(out), _p(ws), ws.numel(), _p(status),
         _stream())
    return out


FFN_DELAYED_GS_H = 1
FFN_DETERMINISTIC = 2


def moe_ffn_forward_ex(x, logits, k, w1: NVFP4Weights, w2: NVFP4Weights, gs_h, delayed=False,
                       deterministic=False, h_stats=None, out=None, ws=None, status=None):
    """moe_ffn_forward with options: h_stats (device int32 (3,), filled: amax bits of |h|,
    saturated and underflowed block scales); delayed=True: gs_h (device float[1]) replaced after
    use by 2688 / amax(h) for the next call; deterministic=True: the slot-ordered output sum."""
    T, H = x.shape
    E = logits.shape[1]
    I = w1.N // 2
    if out is None:
        out = torch.empty(T, H, dtype=BF16, device=x.device)
    need = ffn_workspace_bytes(T, H, I, E, k)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=U8, device=x.device)
    call("moe_ffn_forward_ex", _p(x), _p(logits), T, H, I, E, k, _p(w1.codes), _p(w1.sf),
         _p(w1.gs), _p(w2.codes), _p(w2.sf), _p(w2.gs), _p(gs_h),
         (FFN_DELAYED_GS_H if delayed else 0) | (FFN_DETERMINISTIC if deterministic else 0),
         _p(h_stats), _p(out), _p(ws), ws.numel(), _p(status), _stream())
    return out


def read_status(status):
    """Host copy of a device status word (synchronizes the current stream)."""
    host = torch.zeros(1, dtype=torch.int32)
    rc = lib().nvfp4_read_status(_p(status), host.data_ptr(), _stream())
    return int(host.item()), rc
