"""Back-to-back calls on one stream, sharing one workspace, with no host synchronization between
them: every buffer a call accumulates into (amax word, statistics, the scatter-add accumulator)
must be reset by that call, and nothing one call leaves in the workspace may leak into the next.
Two input sets alternate over many calls; each output must equal the output of the same inputs
computed alone (bitwise on the deterministic paths; for the scatter-add form, whose summation
order is free, within one bf16 ulp per value plus the FP32 reordering error).
"""

import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from tests._gpu_util import DEV

pytestmark = pytest.mark.gpu

ROUNDS = 12


def _weights(E, H, I, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    w1f = [torch.randn(2 * I, H, generator=g).to(torch.bfloat16).to(DEV) for _ in range(E)]
    w2f = [torch.randn(H, I, generator=g).to(torch.bfloat16).to(DEV) for _ in range(E)]
    return nv.quantize_w1(lambda e: w1f[e], E, I, H), nv.quantize_weights(lambda e: w2f[e], E, H, I)


def _inputs(T, H, E, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).to(DEV)
    lg = torch.randn(T, E, generator=g).to(DEV)
    return x, lg


@pytest.mark.parametrize("T", [256, 1024])  # 1024 x 4 slots: the multi-CTA routing
@pytest.mark.parametrize("deterministic", [True, False])
def test_ffn_alternating_inputs(deterministic, T):
    H, I, E, k = 1024, 512, 16, 4  # T*k >= 32*E: the scatter-add form by default
    w1, w2 = _weights(E, H, I, 11)
    gs_h = torch.ones(1, dtype=torch.float32, device=DEV)
    sets = [_inputs(T, H, E, 100 + i) for i in range(2)]
    ws = torch.empty(nv.ffn_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device=DEV)
    alone = []
    for x, lg in sets:
        alone.append(nv.moe_ffn_forward_ex(x, lg, k, w1, w2, gs_h, deterministic=deterministic,
                                           ws=ws))
        torch.cuda.synchronize()
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=DEV) for _ in range(ROUNDS)]
    for r in range(ROUNDS):
        x, lg = sets[r % 2]
        nv.moe_ffn_forward_ex(x, lg, k, w1, w2, gs_h, deterministic=deterministic, out=outs[r],
                              ws=ws)
    torch.cuda.synchronize()
    for r in range(ROUNDS):
        ref = alone[r % 2]
        if deterministic:
            assert torch.equal(outs[r], ref), f"call {r}"
        else:
            # The FP32 sums differ in their last bits (error ~ k * 2^-24 * the largest
            # contribution, bounded here by 2^-16 of the largest output), and the bf16 rounding
            # may then move a value by one ulp (<= 2^-7 of it).  A lost or doubled contribution
            # is of the order of the outputs themselves.
            d = (outs[r].float() - ref.float()).abs()
            tol = ref.float().abs() * 2.0 ** -7 + float(ref.float().abs().max()) * 2.0 ** -16
            bad = d > tol
            i = int(torch.argmax((d - tol).flatten()))
            assert not bool(bad.any()), (
                f"call {r}: {int(bad.sum())} values off, worst |d|={float(d.flatten()[i]):.4g} "
                f"at ref={float(ref.flatten()[i]):.4g} (tol {float(tol.flatten()[i]):.4g})")


def test_linear_split_k_alternating_inputs():
    M, K, N = 16, 2048, 1024  # 4 output tiles: the product is split along K
    g = torch.Generator(device="cpu").manual_seed(5)
    wf = torch.randn(N, K, generator=g).to(torch.bfloat16).to(DEV)
    w = nv.quantize_weights(lambda e: wf, 1, N, K)
    gamma = (torch.rand(K, generator=g) + 0.5).to(torch.bfloat16).to(DEV)
    xs = [torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV) for _ in range(2)]
    ws = torch.empty(max(nv.linear_workspace_bytes(M, N, K), 256), dtype=torch.uint8, device=DEV)
    alone = []
    for x in xs:
        alone.append(nv.linear(x, w, gamma=gamma, ws=ws))
        torch.cuda.synchronize()
    outs = [torch.empty(M, N, dtype=torch.bfloat16, device=DEV) for _ in range(ROUNDS)]
    for r in range(ROUNDS):
        nv.linear(xs[r % 2], w, gamma=gamma, out=outs[r], ws=ws)
    torch.cuda.synchronize()
    for r in range(ROUNDS):
        assert torch.equal(outs[r], alone[r % 2]), f"call {r}"
