"""CPU oracle of the quantised MoE expert forward (fp64, logical layout).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA path; its only common dependency is the seeded input
generator ``synth``.

The arithmetic lives in ``oracle.c`` (plain C, one output at a time); this
module only marshals numpy arrays to it.  Function-by-function citations of
the source pages are in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_OMP_LIB_PATH = os.path.join(_HERE, "liboracle_omp.so")  # timing build: output rows over threads


def _build_one(path: str, extra, force: bool) -> str:
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                               "-ffp-contract=off", *extra, src, "-lm", "-o", path + ".tmp"])
        os.replace(path + ".tmp", path)
    return path


def build(force: bool = False, omp: bool = False) -> str:
    """Builds the plain oracle (the checks use it); with omp, also the
    timing build whose matrix-vector rows run on OpenMP threads."""
    path = _build_one(_LIB_PATH, [], force)
    if omp:
        _build_one(_OMP_LIB_PATH, ["-fopenmp", "-DORACLE_OMP"], force)
    return path


class _Expert(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class _Layer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("G", ctypes.c_int), ("eps", ctypes.c_double), ("w_router", ctypes.c_void_p),
                ("w_shared_gate", ctypes.c_void_p), ("norm_w", ctypes.c_void_p),
                ("experts", ctypes.POINTER(_Expert))]


_lib = None
_libs = {}


def set_threads(n: int) -> int:
    """Timing only (the benchmark's CPU baseline): n > 1 switches every call
    below to the OpenMP build on n threads, n <= 1 back to the plain build.
    Both compute the same values.  Returns the threads in use."""
    global _lib
    if n <= 1:
        _lib = _load(_LIB_PATH)
        return 1
    build(omp=True)
    _lib = _load(_OMP_LIB_PATH)
    _lib.oracle_set_threads(int(n))
    return int(n)


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _load(_LIB_PATH)
    return _lib


def _load(path: str) -> ctypes.CDLL:
    if path not in _libs:
        L = ctypes.CDLL(path)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_bf16.restype = dbl
        L.oracle_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_qgemv.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
        L.oracle_qgemv.restype = None
        L.oracle_gemv_f32.argtypes = [vp, i32, i32, vp, vp, vp]
        L.oracle_gemv_f32.restype = None
        L.oracle_topk_softmax.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_topk_softmax.restype = i32
        L.oracle_sigmoid.argtypes = [dbl]
        L.oracle_sigmoid.restype = dbl
        L.oracle_swiglu.argtypes = [dbl, dbl]
        L.oracle_swiglu.restype = dbl
        L.oracle_expert_ffn.argtypes = [ctypes.POINTER(_Expert), i32, i32, i32, vp] + [vp] * 8
        L.oracle_expert_ffn.restype = None
        L.oracle_combine_rmsnorm.argtypes = [i32, i32, vp, vp, vp, dbl, dbl, vp, vp, dbl, vp, vp, vp, vp]
        L.oracle_combine_rmsnorm.restype = None
        L.oracle_layer_token.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp] + [vp] * 13
        L.oracle_layer_token.restype = i32
        L.oracle_quantize.argtypes = [vp, ctypes.c_size_t, i32, i32, vp, vp, vp]
        L.oracle_quantize.restype = None
        L.oracle_quantize_f32.argtypes = [vp, ctypes.c_size_t, i32, i32, vp, vp, vp]
        L.oracle_quantize_f32.restype = None
        L.oracle_dequantize.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.oracle_dequantize.restype = None
        if path == _OMP_LIB_PATH:
            L.oracle_set_threads.argtypes = [i32]
            L.oracle_set_threads.restype = None
        _libs[path] = L
    return _libs[path]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def bf16(h: int) -> float:
    return lib().oracle_bf16(int(h))


def qgemv(q, s, b, G: int, x):
    """y = W x with W[r][j] = q[r][j] s[r][j/G] + b[r][j/G]; returns (y, S)."""
    q, s, b = _c(q, np.uint8), _c(s, np.uint16), _c(b, np.uint16)
    x = _c(x, np.float64)
    rows, cols = q.shape
    y = np.empty(rows)
    S = np.empty(rows)
    lib().oracle_qgemv(_p(q), _p(s), _p(b), rows, cols, G, _p(x), _p(y), _p(S))
    return y, S


def gemv_f32(W, x):
    W = _c(W, np.float32)
    x = _c(x, np.float64)
    rows, cols = W.shape
    y, S = np.empty(rows), np.empty(rows)
    lib().oracle_gemv_f32(_p(W), rows, cols, _p(x), _p(y), _p(S))
    return y, S


def topk_softmax(logits, k: int):
    """Returns (ids int32[k], p float64[k], nan_seen)."""
    logits = _c(logits, np.float64)
    ids = np.empty(k, np.int32)
    p = np.empty(k)
    nan = lib().oracle_topk_softmax(_p(logits), logits.size, k, _p(ids), _p(p))
    return ids, p, bool(nan)


def sigmoid(z: float) -> float:
    return lib().oracle_sigmoid(float(z))


def swiglu(g: float, u: float) -> float:
    return lib().oracle_swiglu(float(g), float(u))


def _expert_struct(ex) -> _Expert:
    return _Expert(ex.q.ctypes.data, ex.scale.ctypes.data, ex.bias.ctypes.data)


def expert_ffn(ex, H: int, I: int, G: int, x):
    """One expert on x[H]; returns dict g, u, a, y and error scales S_g, S_u, S_a, S_y."""
    x = _c(x, np.float64)
    out = {n: np.empty(I) for n in ("g", "u", "a", "S_g", "S_u", "S_a")}
    out.update({n: np.empty(H) for n in ("y", "S_y")})
    st = _expert_struct(ex)
    lib().oracle_expert_ffn(ctypes.byref(st), H, I, G, _p(x), _p(out["g"]), _p(out["u"]), _p(out["a"]),
                            _p(out["y"]), _p(out["S_g"]), _p(out["S_u"]), _p(out["S_a"]), _p(out["S_y"]))
    return out


def combine_rmsnorm(y, p, gamma: float, h, w, eps: float, S_y=None, S_gamma: float = 0.0):
    """y [(k+1)][H] (shared last), p [k]; returns (h_out, xn_out, S_h, S_xn)."""
    y = _c(y, np.float64)
    k = y.shape[0] - 1
    H = y.shape[1]
    p = _c(p, np.float64)
    h = _c(h, np.float64)
    w = _c(w, np.float32)
    S_y = _c(S_y, np.float64) if S_y is not None else None
    ho, xo, Sh, Sx = (np.empty(H) for _ in range(4))
    lib().oracle_combine_rmsnorm(H, k, _p(y), _p(S_y), _p(p), float(gamma), float(S_gamma), _p(h), _p(w),
                                 float(eps), _p(ho), _p(xo), _p(Sh), _p(Sx))
    return ho, xo, Sh, Sx


@dataclass
class LayerWeights:
    """Logical weights of one layer: router [E][H], shared gate [H], norm [H]
    and experts (mapping slot -> synth.ExpertLogical; slot E is the shared expert)."""

    w_router: np.ndarray
    w_shared_gate: np.ndarray
    norm_w: np.ndarray
    experts: dict


def layer_token(wl, lw: LayerWeights, h, xn, logits_in=None, expert_fn=None):
    """One token through one layer.  `wl` is a synth.Workload.  If logits_in
    (fp32 [E]) is given, routing uses those logits.  Missing selected experts
    are produced by expert_fn(slot) when given.  Returns a dict of every
    intermediate and its error scale."""
    H, I, E, k = wl.hidden, wl.inter, wl.n_experts, wl.top_k
    h = _c(h, np.float64)
    xn = _c(xn, np.float64)
    if logits_in is not None:
        logits_in = _c(logits_in, np.float32)
    if expert_fn is not None:
        # routing first, to know which experts to materialise
        if logits_in is None:
            lg, _ = gemv_f32(lw.w_router, xn)
        else:
            lg = logits_in.astype(np.float64)
        ids, _, _ = topk_softmax(lg, k)
        for s in list(ids) + [E]:
            if int(s) not in lw.experts:
                lw.experts[int(s)] = expert_fn(int(s))
    arr = (_Expert * (E + 1))()
    for s, ex in lw.experts.items():
        arr[s] = _expert_struct(ex)
    W = _c(lw.w_router, np.float32)
    wsg = _c(lw.w_shared_gate, np.float32)
    nw = _c(lw.norm_w, np.float32)
    L = _Layer(H, I, E, k, wl.group, wl.eps, W.ctypes.data, wsg.ctypes.data, nw.ctypes.data, arr)
    out = {
        "logits": np.empty(E), "S_l": np.empty(E), "ids": np.empty(k, np.int32), "p": np.empty(k),
        "gamma": np.empty(1), "S_gamma": np.empty(1), "y": np.empty((k + 1, H)), "S_y": np.empty((k + 1, H)),
        "h": np.empty(H), "xn": np.empty(H), "S_h": np.empty(H), "S_xn": np.empty(H),
    }
    work = np.empty(6 * I)
    rc = lib().oracle_layer_token(ctypes.byref(L), _p(h), _p(xn), _p(logits_in), _p(out["logits"]), _p(out["S_l"]),
                                  _p(out["ids"]), _p(out["p"]), _p(out["gamma"]), _p(out["S_gamma"]), _p(out["y"]),
                                  _p(out["S_y"]), _p(out["h"]), _p(out["xn"]), _p(out["S_h"]), _p(out["S_xn"]),
                                  _p(work))
    if rc < 0:
        raise ValueError("a selected expert's tensors were not supplied")
    out["nan_seen"] = bool(rc == 1)
    out["gamma"] = float(out["gamma"][0])
    out["S_gamma"] = float(out["S_gamma"][0])
    return out


def quantize(w, G: int, bits: int):
    """Group-affine min/max quantiser; returns (q uint8, s float64, b float64)."""
    w = _c(w, np.float64)
    q = np.empty(w.shape, np.uint8)
    s = np.empty(w.size // G)
    b = np.empty(w.size // G)
    lib().oracle_quantize(_p(w), w.size, G, bits, _p(q), _p(s), _p(b))
    return q, s, b


def quantize_f32(w, G: int, bits: int):
    """The stored-format quantiser in fp32 (oracle.c, oracle_quantize_f32):
    returns (q uint8, scale bf16 bits uint16, bias bf16 bits uint16)."""
    w = _c(w, np.float32).ravel()
    n_groups = w.size // G
    q = np.empty(w.size, np.uint8)
    s = np.empty(n_groups, np.uint16)
    b = np.empty(n_groups, np.uint16)
    lib().oracle_quantize_f32(_p(w), n_groups, G, bits, _p(q), _p(s), _p(b))
    return q, s, b


def dequantize(q, s, b, G: int):
    q, s, b = _c(q, np.uint8), _c(s, np.uint16), _c(b, np.uint16)
    rows, cols = q.shape
    w = np.empty((rows, cols))
    lib().oracle_dequantize(_p(q), _p(s), _p(b), rows, cols, G, _p(w))
    return w
