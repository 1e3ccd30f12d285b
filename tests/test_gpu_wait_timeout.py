"""Failure detection without a GPU fault: the persistent kernel's grid
barrier is made unreachable by a corrupted counter in the workspace (a value
that the arrivals wrap around), so every CTA's bounded wait runs out (about
two seconds).  The kernel must set FMOE_STATUS_WAIT_TIMEOUT and return; the
context stays usable, and after re-initialising the workspace the same call
succeeds."""
import numpy as np
import pytest
import torch

import synth
from synth.device import upload_layer

pytestmark = pytest.mark.gpu

fm = pytest.importorskip("quantized_expert_gemv_b200")


def test_unreachable_barrier_times_out_and_recovers():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = synth.Workload(hidden=256, inter=256, n_experts=16)
    lw = upload_layer(wl, 0)
    assert fm.fmoe_fused_supported(lw.desc)
    prev = fm.fmoe_set_fused(True)
    try:
        fm.fmoe_read_status(clear=True)
        x = synth.tokens(wl, 1, stream=61)
        ws = fm.alloc_workspace(lw.desc, 1)
        ws[:4] = torch.tensor([0xFF, 0xFF, 0xFF, 0xFF], dtype=torch.uint8, device="cuda")  # barrier counter 2^32 - 1
        h, xn = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
        fm.fmoe_layer_forward(lw, h, xn, ws)
        torch.cuda.synchronize()
        assert fm.fmoe_read_status(clear=True) & fm.FMOE_STATUS_WAIT_TIMEOUT
        # the context is intact: re-initialise the workspace and run again
        fm.fmoe_workspace_init(ws)
        h2, xn2 = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
        fm.fmoe_layer_forward(lw, h2, xn2, ws)
        torch.cuda.synchronize()
        assert fm.fmoe_read_status(clear=True) == 0
        ws3 = fm.alloc_workspace(lw.desc, 1)
        h3, xn3 = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
        fm.fmoe_layer_forward(lw, h3, xn3, ws3)
        torch.cuda.synchronize()
        assert np.array_equal(h2.cpu().numpy(), h3.cpu().numpy())
        assert np.array_equal(xn2.cpu().numpy(), xn3.cpu().numpy())
    finally:
        fm.fmoe_set_fused(prev)
