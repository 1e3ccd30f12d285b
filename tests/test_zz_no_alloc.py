"""fmoe_layer_forward_noalloc (fixed per-device scratch, no allocation)
against fmoe_layer_forward with a caller workspace.

Both run the same kernels, so two calls in a row (the second reading what
the first wrote) must give bit-identical h and xn, with the persistent
kernel enabled and disabled: at T = 1, at T = 3 (a pair and a single token
through the persistent kernel, or one kernel per step), and at the largest
T the 12 MiB scratch admits (the grouped path).  A T beyond that is
refused on the host before anything is launched.  The file name sorts last
so that the test also runs after everything else in the suite has used the
library.
"""
import numpy as np
import pytest
import torch

import synth
from synth.device import upload_layer

pytestmark = pytest.mark.gpu

fm = pytest.importorskip("quantized_expert_gemv_b200")

SCRATCH_BYTES = 12 << 20
SMALL = synth.Workload(hidden=256, inter=256, n_experts=16)


@pytest.fixture(scope="module")
def small_layer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return upload_layer(SMALL, 0)


def _max_tokens(desc):
    T = 1
    while fm.fmoe_workspace_bytes(desc, T + 1) <= SCRATCH_BYTES:
        T += 1
    return T


def _two_calls(fn, x):
    h = torch.from_numpy(x).cuda()
    xn = torch.from_numpy(x).cuda()
    outs = []
    for _ in range(2):
        fn(h, xn)
        torch.cuda.synchronize()
        outs.append((h.cpu().numpy().copy(), xn.cpu().numpy().copy()))
    return outs


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "per-step"])
@pytest.mark.parametrize("T", [1, 3, "max"])
def test_noalloc_matches_workspace_entry_point(small_layer, T, fused):
    lw = small_layer
    T = _max_tokens(lw.desc) if T == "max" else T
    x = synth.tokens(SMALL, T, stream=71)
    prev = fm.fmoe_set_fused(fused)
    try:
        fm.fmoe_read_status(clear=True)
        ws = fm.alloc_workspace(lw.desc, T)
        ref = _two_calls(lambda h, xn: fm.fmoe_layer_forward(lw, h, xn, ws), x)
        got = _two_calls(lambda h, xn: fm.fmoe_layer_forward_noalloc(lw, h, xn), x)
    finally:
        fm.fmoe_set_fused(prev)
    for i in range(2):
        assert np.array_equal(got[i][0], ref[i][0]), f"h after call {i + 1}"
        assert np.array_equal(got[i][1], ref[i][1]), f"xn after call {i + 1}"
    assert not np.array_equal(ref[0][0], ref[1][0])  # the second call did work on new input
    assert fm.fmoe_read_status() == 0


def test_noalloc_rejects_tokens_beyond_scratch(small_layer):
    lw = small_layer
    T = _max_tokens(lw.desc) + 1
    assert fm.fmoe_workspace_bytes(lw.desc, T) > SCRATCH_BYTES
    h = torch.zeros(T, SMALL.hidden, device="cuda")
    xn = torch.zeros(T, SMALL.hidden, device="cuda")
    with pytest.raises(fm.FmoeError) as e:
        fm.fmoe_layer_forward_noalloc(lw, h, xn)
    assert e.value.status == fm.FMOE_ERR_BUFFER_TOO_SMALL
    assert not h.any() and not xn.any()


def test_noalloc_scratch_shared_across_shapes():
    """One scratch array serves every shape: a many-token call of a small
    layer (whose grouping data land where a larger layer's persistent
    kernel keeps its exchange words, were those placed by shape) followed by
    a single-token call of a larger layer must give the bits of that call on
    a fresh workspace."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    small = upload_layer(SMALL, 0)
    big_wl = synth.Workload(hidden=1024, inter=512, n_experts=64)
    big = upload_layer(big_wl, 0)
    assert fm.fmoe_fused_supported(big.desc)
    fm.fmoe_read_status(clear=True)
    xs = synth.tokens(SMALL, 8, stream=75)
    h, xn = torch.from_numpy(xs).cuda(), torch.from_numpy(xs).cuda()
    fm.fmoe_layer_forward_noalloc(small, h, xn)  # T = 8: the grouped path
    xb = synth.tokens(big_wl, 1, stream=76)
    ws = fm.alloc_workspace(big.desc, 1)
    ref = _two_calls(lambda h, xn: fm.fmoe_layer_forward(big, h, xn, ws), xb)
    got = _two_calls(lambda h, xn: fm.fmoe_layer_forward_noalloc(big, h, xn), xb)
    for i in range(2):
        assert np.array_equal(got[i][0], ref[i][0]) and np.array_equal(got[i][1], ref[i][1]), i
    assert fm.fmoe_read_status() == 0
