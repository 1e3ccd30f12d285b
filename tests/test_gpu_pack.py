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


def _quantiser_inputs(n_groups, seed):
    """fp32 weights of the expert scale (normal, 0.02), plus groups that test
    the edge cases: constant, signed zeros at the minimum, all negative,
    large magnitude, exact code grids, a tiny range."""
    r = np.random.default_rng(seed)
    w = (r.normal(size=(n_groups, 64)) * 0.02).astype(np.float32)
    w[0] = 0.125
    w[1] = r.normal(size=64).astype(np.float32) ** 2
    w[1, :3] = [-0.0, 0.0, -0.0]
    w[2] = -r.uniform(1.0, 2.0, size=64)
    w[3] = r.normal(size=64) * 3e4
    w[4] = (r.integers(0, 16, size=64) * np.float32(2 ** -7) - np.float32(0.5)).astype(np.float32)
    w[5] = np.float32(1.0) + r.uniform(0, 1e-6, size=64).astype(np.float32)
    return w


@pytest.mark.parametrize("bits", [4, 2])
def test_device_quantiser_matches_oracle(bits):
    """Codes, bf16 scales and biases bit for bit against the oracle's fp32
    quantiser, at a full expert's worth of groups."""
    import oracle
    n_groups = 3 * 4096 * 1024 // 64
    w = _quantiser_inputs(n_groups, 40 + bits)
    q_ref, s_ref, b_ref = oracle.quantize_f32(w, 64, bits)
    wd = torch.from_numpy(w).cuda()
    q = torch.empty(w.size, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n_groups, dtype=torch.int16, device="cuda")
    bi = torch.empty(n_groups, dtype=torch.int16, device="cuda")
    fm.fmoe_quantize_groups(wd, bits, q, sc, bi)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), s_ref)
    assert np.array_equal(bi.cpu().numpy().view(np.uint16), b_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("bits", [4, 2])
def test_quantise_then_pack_round_trip(bits):
    """fp32 expert weights -> device quantiser -> device packer; unpacking
    the records on the host gives back the quantiser's codes, scales and
    biases."""
    H, I, E = 256, 128, 3
    n = 3 * H * I * E
    w = _quantiser_inputs(n // 64, 50 + bits).ravel()
    wd = torch.from_numpy(w).cuda()
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n // 64, dtype=torch.int16, device="cuda")
    bi = torch.empty(n // 64, dtype=torch.int16, device="cuda")
    fm.fmoe_quantize_groups(wd, bits, q, sc, bi)
    nbytes = fm.fmoe_packed_bytes(bits, E, H, I, 64)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    fm.fmoe_pack_experts_device(q, sc, bi, bits, E, H, I, packed)
    torch.cuda.synchronize()
    assert fm.fmoe_read_status() == 0
    q2, s2, b2 = fm.fmoe_unpack_experts_host(packed.cpu().numpy(), bits, E, H, I)
    assert np.array_equal(q2.ravel(), q.cpu().numpy())
    assert np.array_equal(s2.ravel(), sc.cpu().numpy().view(np.uint16))
    assert np.array_equal(b2.ravel(), bi.cpu().numpy().view(np.uint16))
