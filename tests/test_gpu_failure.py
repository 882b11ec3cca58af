"""Failure detection on the GPU without a fault: a bounded wait runs out (on an mbarrier that
nothing arrives on), the other waiting role gives up early through the abort flag, the status word
reports NVFP4_DEVERR_TIMEOUT, and the context stays usable for the next kernel."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_gsa_b200 as nv
from nvfp4_block_scaled_gsa_b200._native import lib
from tests._gpu_util import DEV

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    elapsed = torch.zeros(1, dtype=torch.int64, device=DEV)
    limit = 20_000_000  # 20 ms
    rc = lib().nvfp4_wait_selftest(limit, status.data_ptr(), elapsed.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    code, rc = nv.read_status(status)
    assert code & 1 and rc == 6  # NVFP4_DEVERR_TIMEOUT, NVFP4_ERR_TIMEOUT
    ns = int(elapsed.item())
    # the limited wait ran its 20 ms; the second warp (2 s limit) left early on the abort flag
    assert limit <= ns < 500_000_000


def test_context_usable_after_a_timeout():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert lib().nvfp4_wait_selftest(5_000_000, status.data_ptr(), None,
                                     torch.cuda.current_stream().cuda_stream) == 0
    code, _ = nv.read_status(status)
    assert code & 1
    # a quantize round trip afterwards still gives the right codes
    x = torch.tensor(np.linspace(-6, 6, 64, dtype=np.float32)[None].repeat(4, 0),
                     dtype=torch.bfloat16, device=DEV)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    codes, sf, _ = nv.quantize(x, gs=gs)
    torch.cuda.synchronize()
    assert codes.shape == (4, 32) and int(codes.cpu().numpy()[0, -1]) >> 4 == 0x7  # +6 -> 0b0111
