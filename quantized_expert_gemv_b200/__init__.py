"""Quantised MoE expert forward for B200 (sm_100a): Python binding of libfmoe.

A thin ctypes layer over the C ABI declared in include/fmoe.h: it converts
torch tensors / numpy arrays to pointers and checks status codes.  Every step
of the computation runs in the library's CUDA kernels; there is no Python or
CPU fallback.  If libfmoe.so has not been built, importing this package
raises ImportError (build it with ``python quantized_expert_gemv_b200/build.py``
or ``__graft_entry__.build()``).

PyTorch is used only for device memory and streams: device arguments are
CUDA tensors, and work is enqueued on ``torch.cuda.current_stream()`` unless
a stream is given.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libfmoe.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: the CUDA library has not been built "
        "(run `python quantized_expert_gemv_b200/build.py`). There is no fallback.")

_lib = ctypes.CDLL(_LIB_PATH)

FMOE_OK = 0
FMOE_ERR_INVALID_ARG = 1
FMOE_ERR_UNSUPPORTED = 2
FMOE_ERR_CUDA = 3
FMOE_ERR_DEVICE_STATUS = 4
FMOE_ERR_BUFFER_TOO_SMALL = 5

FMOE_STATUS_BAD_EXPERT_ID = 0x1
FMOE_STATUS_NAN_LOGIT = 0x2
FMOE_STATUS_WAIT_TIMEOUT = 0x4
FMOE_STATUS_BAD_PACK_INPUT = 0x8

FMOE_LOGITS_GIVEN = 0x1

WS_LOGITS, WS_IDS, WS_WEIGHTS, WS_GAMMA, WS_A, WS_Y = range(6)
TRACE_XN_IN, TRACE_LOGITS, TRACE_IDS, TRACE_WEIGHTS, TRACE_GAMMA, TRACE_A, TRACE_H_OUT = range(7)

LIBRARY_PATH = _LIB_PATH


class FmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fmoe_error_string(status)} (status {status})")


class fmoe_layer_desc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("bits", ctypes.c_int), ("shared_bits", ctypes.c_int),
                ("group", ctypes.c_int), ("eps", ctypes.c_float)]


class fmoe_layer_weights(ctypes.Structure):
    _fields_ = [("desc", fmoe_layer_desc), ("experts", ctypes.c_void_p), ("shared", ctypes.c_void_p),
                ("w_router", ctypes.c_void_p), ("w_shared_gate", ctypes.c_void_p),
                ("norm_w", ctypes.c_void_p)]


_vp, _i32, _u32, _sz, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_float
_PDESC = ctypes.POINTER(fmoe_layer_desc)
_PW = ctypes.POINTER(fmoe_layer_weights)

_SIGS = {
    "fmoe_error_string": (ctypes.c_char_p, [_i32]),
    "fmoe_read_status": (_i32, [ctypes.POINTER(ctypes.c_uint32), _i32]),
    "fmoe_packed_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "fmoe_pack_experts_host": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _sz]),
    "fmoe_unpack_experts_host": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "fmoe_pack_experts": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "fmoe_pack_experts_device": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "fmoe_workspace_bytes": (_sz, [_PDESC, _i32]),
    "fmoe_workspace_init": (_i32, [_vp, _sz, _vp]),
    "fmoe_workspace_offset": (_sz, [_PDESC, _i32, _i32]),
    "fmoe_route_topk": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _u32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fmoe_expert_forward": (_i32, [_PW, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "fmoe_combine_residual_rmsnorm": (_i32, [_vp, _vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "fmoe_layer_forward": (_i32, [_PW, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_layer_forward_logits": (_i32, [_PW, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_stack_forward": (_i32, [_PW, _i32, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_stack_forward_trace": (_i32, [_PW, _i32, _vp, _vp, _i32, _vp, _sz, _vp, _sz, _vp]),
    "fmoe_trace_bytes": (_sz, [_PDESC, _i32, _i32]),
    "fmoe_trace_offset": (_sz, [_PDESC, _i32, _i32, _i32]),
    "fmoe_set_fused": (_i32, [_i32]),
    "fmoe_fused_supported": (_i32, [_PDESC]),
    "fmoe_set_tensor_cores": (_i32, [_i32]),
    "fmoe_tc_min_tokens": (_i32, []),
    "fmoe_cache_create": (_i32, [_vp, _i32, _vp, _i32, _vp, _sz, _vp, _i32, _vp]),
    "fmoe_cache_destroy": (_i32, [_vp]),
    "fmoe_cache_stats": (_i32, [_vp, _vp, _vp, _vp]),
    "fmoe_cache_layer_forward": (_i32, [_vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_layer_forward_host": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_stack_forward_host": (_i32, [_PW, _i32, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "fmoe_quantize_groups": (_i32, [_vp, _sz, _i32, _i32, _vp, _vp, _vp, _vp]),
    "fmoe_fused_max_tokens": (_i32, [_i32]),
    "fmoe_layer_forward_noalloc": (_i32, [_PW, _vp, _vp, _i32, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _check(rc: int, where: str) -> None:
    if rc != FMOE_OK:
        raise FmoeError(rc, where)


def _ptr(x):
    """Device or host pointer of a torch tensor / numpy array (None -> NULL;
    an int is taken as a raw address)."""
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be contiguous")
        return ctypes.c_void_p(x.ctypes.data)
    if isinstance(x, int):
        return ctypes.c_void_p(x)
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(x.data_ptr())


_DT = {"f32": (np.float32, "float32"), "i32": (np.int32, "int32")}


def _need(x, name: str, n: int, dt: str | None = "f32", cuda: bool = True, exact: bool = True) -> None:
    """Refuses (ValueError) a buffer that a C call would read or write out of
    its bounds, as the wrong element type or in the wrong memory, before the
    call: x must be contiguous, hold exactly (exact) or at least n elements
    of type dt (dt None: n counts bytes, any type), and live on a CUDA device
    (cuda) or in host memory.  Raw int addresses are the caller's own."""
    if isinstance(x, int):
        return
    if x is None:
        raise ValueError(f"{name}: missing")
    if isinstance(x, np.ndarray):
        where, contiguous, size, nbytes = "cpu", x.flags["C_CONTIGUOUS"], x.size, x.nbytes
        dt_ok = dt is None or x.dtype == np.dtype(_DT[dt][0])
    else:
        where, contiguous = x.device.type, x.is_contiguous()
        size, nbytes = x.numel(), x.numel() * x.element_size()
        dt_ok = dt is None or str(x.dtype) == "torch." + _DT[dt][1]
    if where != ("cuda" if cuda else "cpu"):
        raise ValueError(f"{name}: must be in {'CUDA device' if cuda else 'host'} memory")
    if not contiguous:
        raise ValueError(f"{name}: must be contiguous")
    if not dt_ok:
        raise ValueError(f"{name}: must hold {_DT[dt][1]} elements, not {x.dtype}")
    have = size if dt is not None else nbytes
    if (have != n) if exact else (have < n):
        unit = "elements" if dt is not None else "bytes"
        raise ValueError(f"{name}: holds {have} {unit}, the call needs {'' if exact else 'at least '}{n}")


def _tokens(lw_or_desc, h, xn, name_h: str = "h", name_xn: str = "xn") -> int:
    """T of the token buffers h, xn [T][hidden] (fp32, device)."""
    H = lw_or_desc.hidden
    T = int(h.shape[0]) if len(getattr(h, "shape", ())) >= 1 else 0
    _need(h, name_h, T * H)
    _need(xn, name_xn, T * H)
    return T


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def fmoe_error_string(status: int) -> str:
    return _lib.fmoe_error_string(status).decode()


def fmoe_read_status(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.fmoe_read_status(ctypes.byref(v), int(clear)), "fmoe_read_status")
    return int(v.value)


def fmoe_packed_bytes(bits: int, n_experts: int, hidden: int, inter: int, group: int = 64) -> int:
    return int(_lib.fmoe_packed_bytes(bits, n_experts, hidden, inter, group))


def _pack_inputs(q, scale, bias, bits: int, n_experts: int, hidden: int, inter: int, group: int, cuda: bool) -> None:
    """The logical codes (one byte each) and bf16 scale / bias (two bytes
    each, per group) that a packer reads must all be there; checked when the
    shape is one the library packs (otherwise its status says why)."""
    if n_experts < 1 or group < 1 or fmoe_packed_bytes(bits, n_experts, hidden, inter, group) <= 0:
        return
    n = n_experts * 3 * hidden * inter
    _need(q, "q", n, None, cuda=cuda, exact=False)
    _need(scale, "scale", 2 * (n // group), None, cuda=cuda, exact=False)
    _need(bias, "bias", 2 * (n // group), None, cuda=cuda, exact=False)


def fmoe_pack_experts_host(q: np.ndarray, scale: np.ndarray, bias: np.ndarray, bits: int, n_experts: int,
                           hidden: int, inter: int, group: int = 64, out: np.ndarray | None = None) -> np.ndarray:
    _pack_inputs(q, scale, bias, bits, n_experts, hidden, inter, group, cuda=False)
    n = fmoe_packed_bytes(bits, n_experts, hidden, inter, group)
    if out is None:
        out = np.empty(max(n, 1), np.uint8)
    rc = _lib.fmoe_pack_experts_host(_ptr(q), _ptr(scale), _ptr(bias), bits, n_experts, hidden, inter, group,
                                     _ptr(out), out.nbytes)
    _check(rc, "fmoe_pack_experts_host")
    return out


def fmoe_unpack_experts_host(packed: np.ndarray, bits: int, n_experts: int, hidden: int, inter: int,
                             group: int = 64):
    if n_experts >= 1 and fmoe_packed_bytes(bits, n_experts, hidden, inter, group) > 0:
        _need(packed, "packed", fmoe_packed_bytes(bits, n_experts, hidden, inter, group), None, cuda=False,
              exact=False)
    n = hidden * inter
    q = np.empty(n_experts * 3 * n, np.uint8)
    s = np.empty(n_experts * 3 * n // group, np.uint16)
    b = np.empty_like(s)
    rc = _lib.fmoe_unpack_experts_host(_ptr(packed), bits, n_experts, hidden, inter, group, _ptr(q), _ptr(s), _ptr(b))
    _check(rc, "fmoe_unpack_experts_host")
    return q, s, b


def fmoe_pack_experts(q, scale, bias, bits: int, n_experts: int, hidden: int, inter: int, d_packed,
                      group: int = 64, stream=None, byte_offset: int = 0) -> None:
    """Packs host logical experts into the device tensor d_packed (at byte_offset)."""
    _pack_inputs(q, scale, bias, bits, n_experts, hidden, inter, group, cuda=False)
    _need(d_packed, "d_packed", byte_offset, None, exact=False)
    dst = d_packed.data_ptr() + byte_offset
    avail = d_packed.numel() * d_packed.element_size() - byte_offset
    rc = _lib.fmoe_pack_experts(_ptr(q), _ptr(scale), _ptr(bias), bits, n_experts, hidden, inter, group,
                                ctypes.c_void_p(dst), avail, _stream(stream))
    _check(rc, "fmoe_pack_experts")


def fmoe_pack_experts_device(d_q, d_scale, d_bias, bits: int, n_experts: int, hidden: int, inter: int, d_packed,
                             group: int = 64, stream=None, byte_offset: int = 0) -> None:
    """Packs logical experts already on the device into d_packed (at byte_offset)."""
    _pack_inputs(d_q, d_scale, d_bias, bits, n_experts, hidden, inter, group, cuda=True)
    _need(d_packed, "d_packed", byte_offset, None, exact=False)
    dst = d_packed.data_ptr() + byte_offset
    avail = d_packed.numel() * d_packed.element_size() - byte_offset
    rc = _lib.fmoe_pack_experts_device(_ptr(d_q), _ptr(d_scale), _ptr(d_bias), bits, n_experts, hidden, inter,
                                       group, ctypes.c_void_p(dst), avail, _stream(stream))
    _check(rc, "fmoe_pack_experts_device")


@dataclass
class LayerDesc:
    hidden: int = 4096
    inter: int = 1024
    n_experts: int = 512
    top_k: int = 4
    bits: int = 4
    shared_bits: int = 4
    group: int = 64
    eps: float = 1e-6

    def c(self) -> fmoe_layer_desc:
        return fmoe_layer_desc(self.hidden, self.inter, self.n_experts, self.top_k, self.bits,
                               self.shared_bits, self.group, self.eps)

    def record_bytes(self, shared: bool = False) -> int:
        return fmoe_packed_bytes(self.shared_bits if shared else self.bits, 1, self.hidden, self.inter, self.group)


@dataclass
class LayerWeights:
    """Device tensors of one layer (kept alive here) and their C descriptor."""

    desc: LayerDesc
    experts: object        # uint8 CUDA tensor, E packed records
    shared: object         # uint8 CUDA tensor, one packed record
    w_router: object       # fp32 CUDA [E][H]
    w_shared_gate: object  # fp32 CUDA [H]
    norm_w: object         # fp32 CUDA [H]
    _c: fmoe_layer_weights = field(default=None, repr=False)

    def c(self) -> fmoe_layer_weights:
        if self._c is None:
            d = self.desc
            _need(self.experts, "experts", d.n_experts * d.record_bytes(), None, exact=False)
            _need(self.shared, "shared", d.record_bytes(shared=True), None, exact=False)
            _need(self.w_router, "w_router", d.n_experts * d.hidden)
            _need(self.w_shared_gate, "w_shared_gate", d.hidden)
            _need(self.norm_w, "norm_w", d.hidden)
            self._c = fmoe_layer_weights(self.desc.c(), self.experts.data_ptr(), self.shared.data_ptr(),
                                         self.w_router.data_ptr(), self.w_shared_gate.data_ptr(),
                                         self.norm_w.data_ptr())
        return self._c


def fmoe_workspace_bytes(desc: LayerDesc, T: int) -> int:
    d = desc.c()
    return int(_lib.fmoe_workspace_bytes(ctypes.byref(d), T))


def fmoe_workspace_init(ws, stream=None) -> None:
    _check(_lib.fmoe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "fmoe_workspace_init")


def fmoe_workspace_offset(desc: LayerDesc, T: int, which: int) -> int:
    d = desc.c()
    return int(_lib.fmoe_workspace_offset(ctypes.byref(d), T, which))


def alloc_workspace(desc: LayerDesc, T: int, device="cuda"):
    """A zero-initialised workspace tensor (uint8) for T tokens."""
    import torch
    n = fmoe_workspace_bytes(desc, T)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def workspace_view(ws, desc: LayerDesc, T: int, which: int):
    """Typed view of an intermediate that fmoe_layer_forward leaves in the workspace."""
    import torch
    k, H, I, E = desc.top_k, desc.hidden, desc.inter, desc.n_experts
    off = fmoe_workspace_offset(desc, T, which)
    shapes = {WS_LOGITS: ((T, E), torch.float32), WS_IDS: ((T, k), torch.int32),
              WS_WEIGHTS: ((T, k), torch.float32), WS_GAMMA: ((T,), torch.float32),
              WS_A: ((T, k + 1, I), torch.float32), WS_Y: ((T, k + 1, H), torch.float32)}
    shape, dt = shapes[which]
    n = int(np.prod(shape))
    return ws[off:off + 4 * n].view(dt).view(*shape)


def fmoe_route_topk(xn, w_router, k: int, logits, ids, weights, ws=None, flags: int = 0, stream=None) -> None:
    T, E = logits.shape
    H = w_router.shape[1] if w_router is not None else 64
    _need(logits, "logits", T * E)
    _need(ids, "ids", T * k, "i32")
    _need(weights, "weights", T * k)
    if not flags & FMOE_LOGITS_GIVEN:
        _need(w_router, "w_router", E * H)
        _need(xn, "xn", T * H)
        _need(ws, "ws", 0, None, exact=False)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    rc = _lib.fmoe_route_topk(_ptr(xn), _ptr(w_router), T, H, E, k, flags, _ptr(logits), _ptr(ids),
                              _ptr(weights), _ptr(ws), nbytes, _stream(stream))
    _check(rc, "fmoe_route_topk")


def fmoe_expert_forward(lw: LayerWeights, xn, ids, y, gamma, ws, stream=None) -> None:
    T = xn.shape[0]
    k, H = lw.desc.top_k, lw.desc.hidden
    _need(xn, "xn", T * H)
    _need(ids, "ids", T * k, "i32")
    _need(y, "y", T * (k + 1) * H)
    _need(gamma, "gamma", T)
    _need(ws, "ws", 0, None, exact=False)
    c = lw.c()
    rc = _lib.fmoe_expert_forward(ctypes.byref(c), _ptr(xn), T, _ptr(ids), lw.desc.top_k, _ptr(y), _ptr(gamma),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "fmoe_expert_forward")


def fmoe_combine_residual_rmsnorm(y, weights, gamma, h, norm_w, eps: float, h_out, xn_out, stream=None) -> None:
    T, k1, H = y.shape
    _need(y, "y", T * k1 * H)
    _need(weights, "weights", T * (k1 - 1))
    _need(gamma, "gamma", T)
    _need(norm_w, "norm_w", H)
    for name, t in (("h", h), ("h_out", h_out), ("xn_out", xn_out)):
        _need(t, name, T * H)
    rc = _lib.fmoe_combine_residual_rmsnorm(_ptr(y), _ptr(weights), _ptr(gamma), _ptr(h), _ptr(norm_w), eps, T,
                                            k1 - 1, H, _ptr(h_out), _ptr(xn_out), _stream(stream))
    _check(rc, "fmoe_combine_residual_rmsnorm")


def fmoe_layer_forward(lw: LayerWeights, h, xn, ws, stream=None) -> None:
    T = _tokens(lw.desc, h, xn)
    _need(ws, "ws", 0, None, exact=False)
    c = lw.c()
    rc = _lib.fmoe_layer_forward(ctypes.byref(c), _ptr(h), _ptr(xn), T, _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "fmoe_layer_forward")


def fmoe_layer_forward_host(lw: LayerWeights, hx_in, hx_out, d_hx, ws, stream=None) -> None:
    """fmoe_layer_forward on host token state: hx_in / hx_out are (pinned) host
    tensors [2, T, H] (h rows, then xn rows), d_hx a device tensor of the same
    shape; one copy in, the layer, one copy out, asynchronous on `stream`."""
    T = int(d_hx.shape[1])
    n = 2 * T * lw.desc.hidden
    _need(d_hx, "d_hx", n)
    _need(hx_in, "hx_in", n, cuda=False)
    _need(hx_out, "hx_out", n, cuda=False)
    _need(ws, "ws", 0, None, exact=False)
    c = lw.c()
    rc = _lib.fmoe_layer_forward_host(ctypes.byref(c), _ptr(hx_in), _ptr(hx_out), _ptr(d_hx), T, _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "fmoe_layer_forward_host")


def fmoe_layer_forward_logits(lw: LayerWeights, logits, h, xn, ws, stream=None) -> None:
    T = _tokens(lw.desc, h, xn)
    _need(logits, "logits", T * lw.desc.n_experts)
    _need(ws, "ws", 0, None, exact=False)
    c = lw.c()
    rc = _lib.fmoe_layer_forward_logits(ctypes.byref(c), _ptr(logits), _ptr(h), _ptr(xn), T, _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "fmoe_layer_forward_logits")


def fmoe_stack_forward_host(layers, hx_in, hx_out, d_hx, ws, stream=None) -> None:
    """fmoe_stack_forward on host token state: hx_in / hx_out (pinned) host
    tensors [2, T, H], d_hx a device tensor of the same shape; one copy in,
    the layers, one copy out, asynchronous on `stream`."""
    T = int(d_hx.shape[1])
    n = 2 * T * layers[0].desc.hidden
    _need(d_hx, "d_hx", n)
    _need(hx_in, "hx_in", n, cuda=False)
    _need(hx_out, "hx_out", n, cuda=False)
    _need(ws, "ws", 0, None, exact=False)
    arr = (fmoe_layer_weights * len(layers))(*[lw.c() for lw in layers])
    rc = _lib.fmoe_stack_forward_host(arr, len(layers), _ptr(hx_in), _ptr(hx_out), _ptr(d_hx), T,
                                      _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "fmoe_stack_forward_host")


def fmoe_stack_forward(layers, h, xn, ws, stream=None, trace=None) -> None:
    """The layer stack in place on h / xn; with `trace` (from alloc_trace),
    fmoe_stack_forward_trace: every layer's input, intermediates and output."""
    T = _tokens(layers[0].desc, h, xn)
    _need(ws, "ws", 0, None, exact=False)
    if trace is not None:
        _need(trace, "trace", 0, None, exact=False)
    arr = (fmoe_layer_weights * len(layers))(*[lw.c() for lw in layers])
    if trace is None:
        rc = _lib.fmoe_stack_forward(arr, len(layers), _ptr(h), _ptr(xn), T, _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream))
        _check(rc, "fmoe_stack_forward")
        return
    rc = _lib.fmoe_stack_forward_trace(arr, len(layers), _ptr(h), _ptr(xn), T, _ptr(ws),
                                       ws.numel() * ws.element_size(), _ptr(trace),
                                       trace.numel() * trace.element_size(), _stream(stream))
    _check(rc, "fmoe_stack_forward_trace")


def fmoe_trace_bytes(desc: LayerDesc, T: int, n_layers: int) -> int:
    d = desc.c()
    return int(_lib.fmoe_trace_bytes(ctypes.byref(d), T, n_layers))


def alloc_trace(desc: LayerDesc, T: int, n_layers: int, device="cuda"):
    """A device buffer (uint8) for the trace of n_layers layers of T tokens."""
    import torch
    return torch.zeros(fmoe_trace_bytes(desc, T, n_layers), dtype=torch.uint8, device=device)


def trace_view(trace, desc: LayerDesc, T: int, layer: int, which: int):
    """Typed view of section `which` (TRACE_*) of layer `layer`'s record."""
    import torch
    k, H, I, E = desc.top_k, desc.hidden, desc.inter, desc.n_experts
    d = desc.c()
    off = int(_lib.fmoe_trace_offset(ctypes.byref(d), T, layer, which))
    shapes = {TRACE_XN_IN: ((T, H), torch.float32), TRACE_LOGITS: ((T, E), torch.float32),
              TRACE_IDS: ((T, k), torch.int32), TRACE_WEIGHTS: ((T, k), torch.float32),
              TRACE_GAMMA: ((T,), torch.float32), TRACE_A: ((T, k + 1, I), torch.float32),
              TRACE_H_OUT: ((T, H), torch.float32)}
    shape, dt = shapes[which]
    n = int(np.prod(shape))
    return trace[off:off + 4 * n].view(dt).view(*shape)


def fmoe_layer_forward_noalloc(lw: LayerWeights, h, xn, stream=None) -> None:
    """fmoe_layer_forward with the library's fixed per-device scratch instead of a
    caller workspace (nothing is allocated; calls on one device must not overlap)."""
    T = _tokens(lw.desc, h, xn)
    c = lw.c()
    rc = _lib.fmoe_layer_forward_noalloc(ctypes.byref(c), _ptr(h), _ptr(xn), T, _stream(stream))
    _check(rc, "fmoe_layer_forward_noalloc")


def fmoe_fused_supported(desc: LayerDesc) -> bool:
    """True if the persistent kernel runs layers of this shape at T = 1 on the current device."""
    c = desc.c() if hasattr(desc, "c") else desc
    return bool(_lib.fmoe_fused_supported(ctypes.byref(c)))


def fmoe_set_tensor_cores(enable: bool) -> bool:
    """Selects tensor-core products (True, default) or the integer-dot path for the
    heavily routed experts of the T > 1 path; returns the previous setting."""
    return bool(_lib.fmoe_set_tensor_cores(int(bool(enable))))


def fmoe_quantize_groups(w, bits: int, q, scale, bias, stream=None) -> None:
    """Quantises the fp32 device tensor w (64-value groups, contiguous) into
    codes q (uint8, one per value) and bf16 bit patterns scale, bias (int16 or
    uint16 tensors, one per group), caller-allocated."""
    n = w.numel()
    if n % 64:
        raise ValueError("w must hold whole 64-value groups")
    _need(w, "w", n)
    _need(q, "q", n, None, exact=False)
    _need(scale, "scale", 2 * (n // 64), None, exact=False)
    _need(bias, "bias", 2 * (n // 64), None, exact=False)
    rc = _lib.fmoe_quantize_groups(_ptr(w), n // 64, 64, bits, _ptr(q), _ptr(scale), _ptr(bias), _stream(stream))
    _check(rc, "fmoe_quantize_groups")


def fmoe_tc_min_tokens() -> int:
    """Tokens an expert needs in a step for the tensor-core products."""
    return int(_lib.fmoe_tc_min_tokens())


def fmoe_fused_max_tokens(stack: bool = False) -> int:
    """Largest T that runs through the persistent kernel (layer or stack call), two tokens per launch."""
    return int(_lib.fmoe_fused_max_tokens(int(bool(stack))))


def fmoe_set_fused(enable: bool) -> bool:
    """Selects the persistent fused kernel (True, default) or the one-kernel-per-step
    path for T = 1; returns the previous setting."""
    return bool(_lib.fmoe_set_fused(int(bool(enable))))


class ExpertCache:
    """Routed experts of n layers in host memory, a device cache of n_slots
    records (C ABI fmoe_cache_*).  host_layers: per layer a (pinned) uint8
    CPU tensor of the layer's E packed records; the device slots and the
    record table are allocated here, as caller-owned buffers of the ABI."""

    def __init__(self, desc: LayerDesc, host_layers, n_slots: int, max_tokens: int = 64):
        import torch
        self.desc, self.host_layers = desc, list(host_layers)
        rec = desc.record_bytes()
        for l, t in enumerate(self.host_layers):
            _need(t, f"host_layers[{l}]", desc.n_experts * rec, None, cuda=False, exact=False)
        self.slots = torch.empty(n_slots * rec, dtype=torch.uint8, device="cuda")
        self.table = torch.zeros(len(self.host_layers) * desc.n_experts, dtype=torch.int64, device="cuda")
        ptrs = (ctypes.c_void_p * len(self.host_layers))(*[t.data_ptr() for t in self.host_layers])
        h = ctypes.c_void_p()
        d = desc.c()
        rc = _lib.fmoe_cache_create(ctypes.byref(d), len(self.host_layers), ptrs, n_slots, _ptr(self.slots),
                                    self.slots.numel(), _ptr(self.table), max_tokens, ctypes.byref(h))
        _check(rc, "fmoe_cache_create")
        self._h = h

    def forward(self, layer: int, lw: LayerWeights, h, xn, ws, logits=None, stream=None) -> None:
        T = _tokens(lw.desc, h, xn)
        _need(ws, "ws", 0, None, exact=False)
        if logits is not None:
            _need(logits, "logits", T * lw.desc.n_experts)
        c = self._weights(lw)
        rc = _lib.fmoe_cache_layer_forward(self._h, layer, ctypes.byref(c), _ptr(logits) if logits is not None else None,
                                           _ptr(h), _ptr(xn), T, _ptr(ws), ws.numel() * ws.element_size(),
                                           _stream(stream))
        _check(rc, "fmoe_cache_layer_forward")

    @staticmethod
    def _weights(lw: LayerWeights) -> fmoe_layer_weights:
        """The C descriptor of lw for a cached layer: its routed records come
        from the cache, so lw.experts may be None (it is not read); the other
        buffers are checked as for a resident layer."""
        d = lw.desc
        _need(lw.shared, "shared", d.record_bytes(shared=True), None, exact=False)
        _need(lw.w_router, "w_router", d.n_experts * d.hidden)
        _need(lw.w_shared_gate, "w_shared_gate", d.hidden)
        _need(lw.norm_w, "norm_w", d.hidden)
        return fmoe_layer_weights(d.c(), lw.experts.data_ptr() if lw.experts is not None else None,
                                  lw.shared.data_ptr(), lw.w_router.data_ptr(), lw.w_shared_gate.data_ptr(),
                                  lw.norm_w.data_ptr())

    def stats(self):
        hits, misses, nbytes = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
        _check(_lib.fmoe_cache_stats(self._h, ctypes.byref(hits), ctypes.byref(misses), ctypes.byref(nbytes)),
               "fmoe_cache_stats")
        return hits.value, misses.value, nbytes.value

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.fmoe_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
