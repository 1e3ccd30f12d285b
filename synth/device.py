"""Device-side synthetic layers: generation on the GPU and upload through the
library's packer.

Used by the GPU tests and the benchmark (never by the oracle).  Logical
tensors come from the generator of this package -- on the host (synth.c) or
on the device (synth_device.cu, the same streams, byte for byte) -- and the
packed device layout from ``quantized_expert_gemv_b200``'s packer.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import (K_BIAS, K_CODES, K_SCALE, LAYER, Workload, _DEV_LIB_PATH, build, expert, key,
               norm_weight, router, shared_gate)

_dlib = None


def dlib() -> ctypes.CDLL:
    global _dlib
    if _dlib is None:
        build(device=True)
        L = ctypes.CDLL(_DEV_LIB_PATH)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.synth_dev_codes.argtypes = [u64, i32, u64, vp, vp]
        L.synth_dev_codes.restype = i32
        L.synth_dev_scale_bias.argtypes = [u64, u64, i32, dbl, dbl, dbl, u64, vp, vp, vp]
        L.synth_dev_scale_bias.restype = i32
        _dlib = L
    return _dlib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def expert_to_device(wl: Workload, layer: int, slot: int, q, s, b) -> None:
    """Generates expert `slot` of `layer` straight into device tensors q (uint8,
    3 H I), s and b (int16/uint16 views, 3 H I / 64), as synth.expert does on the host."""
    L = dlib()
    bits = wl.expert_bits(slot)
    n = wl.hidden * wl.inter
    ng = n // wl.group
    lo, hi = wl.scale_range(bits)
    st = _stream()
    for m in range(3):
        rc = L.synth_dev_codes(key(wl.seed, K_CODES[m], layer, slot), bits, n,
                               ctypes.c_void_p(q.data_ptr() + m * n), st)
        assert rc == 0, rc
        rc = L.synth_dev_scale_bias(key(wl.seed, K_SCALE[m], layer, slot), key(wl.seed, K_BIAS[m], layer, slot),
                                    bits, lo, hi, wl.bias_sigma, ng, ctypes.c_void_p(s.data_ptr() + 2 * m * ng),
                                    ctypes.c_void_p(b.data_ptr() + 2 * m * ng), st)
        assert rc == 0, rc


def layer_desc(wl: Workload):
    import quantized_expert_gemv_b200 as fm
    return fm.LayerDesc(wl.hidden, wl.inter, wl.n_experts, wl.top_k, wl.bits, wl.shared_bits, wl.group, wl.eps)


def upload_layer(wl: Workload, layer: int, device="cuda", chunk: int = 32, scratch=None):
    """All E routed experts, the shared expert, router, shared gate and norm
    weight of `layer`, generated and packed on the device.  Returns a
    quantized_expert_gemv_b200.LayerWeights.  `scratch` (optional) is a
    reusable dict of logical staging tensors."""
    import torch
    import quantized_expert_gemv_b200 as fm
    desc = layer_desc(wl)
    H, I, E = wl.hidden, wl.inter, wl.n_experts
    n, ng = 3 * H * I, 3 * H * I // wl.group
    chunk = max(1, min(chunk, E))
    if scratch is None:
        scratch = {}
    if scratch.get("n", 0) < chunk * n:
        scratch["q"] = torch.empty(chunk * n, dtype=torch.uint8, device=device)
        scratch["s"] = torch.empty(chunk * ng, dtype=torch.int16, device=device)
        scratch["b"] = torch.empty(chunk * ng, dtype=torch.int16, device=device)
        scratch["n"] = chunk * n
    q, s, b = scratch["q"], scratch["s"], scratch["b"]
    rec = desc.record_bytes()
    experts_t = torch.empty(E * rec, dtype=torch.uint8, device=device)
    for e0 in range(0, E, chunk):
        ne = min(chunk, E - e0)
        for i in range(ne):
            expert_to_device(wl, layer, e0 + i, q[i * n:(i + 1) * n], s[i * ng:(i + 1) * ng], b[i * ng:(i + 1) * ng])
        fm.fmoe_pack_experts_device(q, s, b, wl.bits, ne, H, I, experts_t, byte_offset=e0 * rec)
    shared_t = torch.empty(desc.record_bytes(shared=True), dtype=torch.uint8, device=device)
    expert_to_device(wl, layer, E, q[:n], s[:ng], b[:ng])
    fm.fmoe_pack_experts_device(q, s, b, wl.shared_bits, 1, H, I, shared_t)
    torch.cuda.current_stream().synchronize()
    return fm.LayerWeights(desc, experts_t, shared_t,
                           torch.from_numpy(router(wl, layer)).to(device),
                           torch.from_numpy(shared_gate(wl, layer)).to(device),
                           torch.from_numpy(norm_weight(wl, layer)).to(device))


def upload_layer_host(wl: Workload, layer: int, device="cuda", chunk: int = 16):
    """As upload_layer, generating and packing on the host (slow path, used to
    cross-check the device generator and packer)."""
    import torch
    import quantized_expert_gemv_b200 as fm
    from . import ExpertLogical
    desc = layer_desc(wl)
    H, I, E = wl.hidden, wl.inter, wl.n_experts
    n, ng = 3 * H * I, 3 * H * I // wl.group
    rec = desc.record_bytes()
    experts_t = torch.empty(E * rec, dtype=torch.uint8, device=device)
    for e0 in range(0, E, chunk):
        ne = min(chunk, E - e0)
        qh = np.empty(ne * n, np.uint8)
        sh = np.empty(ne * ng, np.uint16)
        bh = np.empty(ne * ng, np.uint16)
        for i in range(ne):
            expert(wl, layer, e0 + i, ExpertLogical(wl.bits, qh[i * n:(i + 1) * n], sh[i * ng:(i + 1) * ng],
                                                     bh[i * ng:(i + 1) * ng]))
        fm.fmoe_pack_experts(qh, sh, bh, wl.bits, ne, H, I, experts_t, byte_offset=e0 * rec)
    ex = expert(wl, layer, E)
    shared_t = torch.empty(desc.record_bytes(shared=True), dtype=torch.uint8, device=device)
    fm.fmoe_pack_experts(ex.q, ex.scale, ex.bias, wl.shared_bits, 1, H, I, shared_t)
    return fm.LayerWeights(desc, experts_t, shared_t,
                           torch.from_numpy(router(wl, layer)).to(device),
                           torch.from_numpy(shared_gate(wl, layer)).to(device),
                           torch.from_numpy(norm_weight(wl, layer)).to(device))


__all__ = ["layer_desc", "upload_layer", "upload_layer_host", "expert_to_device", "LAYER"]
