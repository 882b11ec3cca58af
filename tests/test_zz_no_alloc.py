"""The no-allocation L2 entry point against the allocating one.

moe_grouped_gemm_l2_scatter_noalloc serves callers that cannot allocate device scratch memory (a
runtime that owns all device memory from start-up, or a foreign-language caller that only holds
its inputs and outputs).  Its FP32 per-slot buffer is a static device array inside the library,
so it must give the same bf16 output as moe_grouped_gemm_l2_scatter, which takes that buffer
from the caller.  Two calls in a row also show that nothing carries over from the previous call
through the shared array.

This file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from nvfp4_block_scaled_gsa_b200._native import call, lib
from oracle import moe as M
from oracle import quant as Q
from oracle import routing as R
from synth import CONFIGS, gen_weight_expert, gen_x
from tests._gpu_util import DEV, rel_fro, to_dev, upload_nvfp4

pytestmark = pytest.mark.gpu


def _l2_problem(T=40, H=512, I=256, E=6, k=3, seed=5):
    x = gen_x(CONFIGS["tiny"], T=T, H=H).float().numpy()
    lg = torch.randn(T, E, generator=torch.Generator().manual_seed(seed)).numpy()
    ids, w = R.route_topk(lg, k)
    w1 = M.QuantWeights.from_float(
        np.stack([gen_weight_expert(seed, 1, e, 2 * I, H).float().numpy() for e in range(E)]))
    wf2 = np.stack([gen_weight_expert(seed, 2, e, H, I).float().numpy() for e in range(E)])
    w2 = M.QuantWeights.from_float(wf2)
    gs_h = np.float32(64.0)
    ref = M.moe_ffn(x, None, k, w1, w2, gs_h, ids=ids, weights=w.astype(np.float32).astype(np.float64),
                    keep=True)
    perm = ref["perm"]
    h, sfh = upload_nvfp4(ref["h_codes"], ref["h_sf"])
    w2d = nv.NVFP4Weights(to_dev(w2.codes.reshape(E * H, I // 2)),
                          to_dev(Q.tile_sf(w2.sf.reshape(E * H, I // 16))), to_dev(w2.gs), E, H, I)
    return dict(h=h, sfh=sfh, gs_h=to_dev(np.array([gs_h], np.float32)), w2=w2d,
                offs=to_dev(perm["offs"].astype(np.int32)),
                row_slot=to_dev(perm["row_slot"].astype(np.int32)),
                row_w=to_dev(perm["row_w"].astype(np.float32)),
                dst_row=to_dev(perm["dst_row"].reshape(-1).astype(np.int32)), T=T, k=k, R=perm["R"],
                ref=ref["out"])


def _noalloc(p, out, status):
    w2 = p["w2"]
    call("moe_grouped_gemm_l2_scatter_noalloc", p["h"].data_ptr(), p["sfh"].data_ptr(),
         p["gs_h"].data_ptr(), w2.codes.data_ptr(), w2.sf.data_ptr(), w2.gs.data_ptr(),
         p["offs"].data_ptr(), p["row_slot"].data_ptr(), p["row_w"].data_ptr(),
         p["dst_row"].data_ptr(), w2.E, w2.N, w2.K, p["T"], p["k"], p["R"], out.data_ptr(),
         status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_l2_matches_allocating_entry_point_twice():
    p = _l2_problem()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _, want = nv.l2_scatter(p["h"], p["sfh"], p["gs_h"], p["w2"], p["offs"], p["row_slot"],
                            p["row_w"], p["dst_row"], p["T"], p["k"], status=status)
    outs = []
    for _ in range(2):
        out = torch.empty(p["T"], p["w2"].N, dtype=torch.bfloat16, device=DEV)
        _noalloc(p, out, status)
        outs.append(out)
    torch.cuda.synchronize()
    code, rc = nv.read_status(status)
    assert code == 0 and rc == 0
    w = want.float().cpu().numpy()
    for out in outs:
        got = out.float().cpu().numpy()
        # same kernels, fixed summation order: bitwise equal to the allocating entry point
        assert torch.equal(out.cpu(), want.cpu())
        assert rel_fro(got, M.bf16_round(p["ref"])) <= 1e-3


def test_noalloc_l2_rejects_sizes_beyond_the_static_scratch():
    p = _l2_problem()
    too_many_tokens = (1 << 20) // (p["k"] * p["w2"].N) + 1
    out = torch.empty(1, dtype=torch.bfloat16, device=DEV)
    rc = lib().moe_grouped_gemm_l2_scatter_noalloc(
        p["h"].data_ptr(), p["sfh"].data_ptr(), p["gs_h"].data_ptr(), p["w2"].codes.data_ptr(),
        p["w2"].sf.data_ptr(), p["w2"].gs.data_ptr(), p["offs"].data_ptr(),
        p["row_slot"].data_ptr(), p["row_w"].data_ptr(), p["dst_row"].data_ptr(), p["w2"].E,
        p["w2"].N, p["w2"].K, too_many_tokens, p["k"], p["R"], out.data_ptr(), None,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 4
    assert b"static FP32 scratch" in lib().nvfp4_last_error()
