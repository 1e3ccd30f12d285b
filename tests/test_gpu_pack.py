"""Device-side generation and packing reproduce the host ones byte for byte."""
import numpy as np
import pytest
import torch

import synth
from synth.device import expert_to_device

pytestmark = pytest.mark.gpu

fm = pytest.importorskip("quantized_expert_gemv_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("wl,slots", [(synth.TINY, [0, 5, 16]),
                                      (synth.Workload(hidden=256, inter=128, n_experts=16, bits=2), [1, 16]),
                                      (synth.LAYER, [0, 311, 512]),
                                      (synth.Workload(bits=2), [7, 512])])
def test_device_generator_matches_host(wl, slots):
    n, ng = 3 * wl.hidden * wl.inter, 3 * wl.hidden * wl.inter // 64
    for slot in slots:
        q = torch.empty(n, dtype=torch.uint8, device="cuda")
        s = torch.empty(ng, dtype=torch.int16, device="cuda")
        b = torch.empty(ng, dtype=torch.int16, device="cuda")
        expert_to_device(wl, 3, slot, q, s, b)
        ref = synth.expert(wl, 3, slot)
        assert np.array_equal(q.cpu().numpy(), ref.q)
        assert np.array_equal(s.cpu().numpy().view(np.uint16), ref.scale)
        assert np.array_equal(b.cpu().numpy().view(np.uint16), ref.bias)


@pytest.mark.parametrize("bits,H,I", [(4, 256, 128), (2, 256, 128), (4, 4096, 1024), (2, 4096, 1024),
                                      (4, 64, 2048), (2, 2048, 64)])
def test_device_packer_matches_host(bits, H, I):
    wl = synth.Workload(hidden=H, inter=I, n_experts=4, bits=bits, seed=3)
    exs = [synth.expert(wl, 0, e) for e in range(3)]
    q = np.concatenate([e.q for e in exs])
    s = np.concatenate([e.scale for e in exs])
    b = np.concatenate([e.bias for e in exs])
    ref = fm.fmoe_pack_experts_host(q, s, b, bits, 3, H, I)
    out = torch.zeros(ref.nbytes, dtype=torch.uint8, device="cuda")
    fm.fmoe_pack_experts_device(torch.from_numpy(q).cuda(), torch.from_numpy(s.view(np.int16)).cuda(),
                                torch.from_numpy(b.view(np.int16)).cuda(), bits, 3, H, I, out)
    assert fm.fmoe_read_status(clear=True) == 0
    assert np.array_equal(out.cpu().numpy(), ref)
    # the host-packer path through the device gives the same bytes too
    out2 = torch.zeros(ref.nbytes, dtype=torch.uint8, device="cuda")
    fm.fmoe_pack_experts(q, s, b, bits, 3, H, I, out2)
    assert np.array_equal(out2.cpu().numpy(), ref)


def test_device_packer_flags_bad_codes():
    H, I = 64, 64
    n, ng = 3 * H * I, 3 * H * I // 64
    q = torch.zeros(n, dtype=torch.uint8, device="cuda")
    q[10] = 17
    s = torch.full((ng,), 0x3F80, dtype=torch.int16, device="cuda")
    b = torch.zeros(ng, dtype=torch.int16, device="cuda")
    out = torch.zeros(fm.fmoe_packed_bytes(4, 1, H, I), dtype=torch.uint8, device="cuda")
    fm.fmoe_read_status(clear=True)
    fm.fmoe_pack_experts_device(q, s, b, 4, 1, H, I, out)
    assert fm.fmoe_read_status(clear=True) & fm.FMOE_STATUS_BAD_PACK_INPUT
