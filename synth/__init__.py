"""Seeded synthetic inputs for the quantised MoE expert forward.

Shared by the CUDA path's tests and benchmark and by the CPU oracle; holds
none of the method's arithmetic.  Every tensor is a pure function of
(seed, kind, layer, slot, element index), computed by the counter-based
generator in ``synth.c`` (SplitMix64 output function), so any expert of any
layer can be regenerated on demand and in parallel.

Workload recipes (the layer shapes and value distributions used throughout):

* ``tiny``   hidden 256, expert intermediate 128, 16 routed experts, top-4,
  one shared expert (intermediate 128), 4-bit codes.
* ``layer``  hidden 4096, expert intermediate 1024, 512 routed experts,
  top-4, one shared expert (intermediate 1024), 4-bit codes.
* ``int2``   the ``layer`` shape with 2-bit routed experts; the shared
  expert keeps 4-bit codes.

Distributions: 4-bit codes U{0..15}, 2-bit codes U{0..3}; group 64 along
the input dimension; bf16 scale U(0.005, 0.02) (4-bit) or U(0.02, 0.08)
(2-bit); bias bf16(-8 s + N(0, 1e-3)) (4-bit) or bf16(-1.5 s) (2-bit);
x ~ N(0, 1) fp32; router rows and the shared-expert gate vector
~ N(0, 0.02) fp32; RMSNorm weight ~ 1 + N(0, 0.1) fp32; eps 1e-6.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

# stream kinds
K_CODES = (1, 2, 3)  # gate, up, down
K_SCALE = (4, 5, 6)
K_BIAS = (7, 8, 9)
K_ROUTER = 10
K_SHARED_GATE = 11
K_NORM = 12
K_X = 13
K_ZIPF_PERM = 14
K_GUMBEL = 15
K_RESID = 16


_DEV_LIB_PATH = os.path.join(_HERE, "libsynth_cuda.so")


def build(force: bool = False, device: bool = True) -> str:
    """Compile libsynth.so with gcc (plain C) and, when `device`, its CUDA twin
    libsynth_cuda.so with nvcc (sm_100a)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", src, "-lm",
             "-o", _LIB_PATH + ".tmp"]
        )
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    dsrc = os.path.join(_HERE, "synth_device.cu")
    if device and (force or not os.path.exists(_DEV_LIB_PATH)
                   or os.path.getmtime(_DEV_LIB_PATH) < os.path.getmtime(dsrc)):
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                               "--shared", "-Xcompiler", "-fPIC", "-fmad=false", dsrc,
                               "-o", _DEV_LIB_PATH + ".tmp"])
        os.replace(_DEV_LIB_PATH + ".tmp", _DEV_LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build(device=False)
        L = ctypes.CDLL(_LIB_PATH)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.synth_key.restype = u64
        L.synth_key.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        L.synth_words.argtypes = [u64, u64, u64, vp]
        L.synth_codes.argtypes = [u64, i32, u64, u64, vp]
        L.synth_scale_bias.argtypes = [u64, u64, i32, dbl, dbl, dbl, u64, u64, vp, vp]
        L.synth_normal_f32.argtypes = [u64, dbl, dbl, u64, u64, vp]
        L.synth_zipf_gumbel_logits.argtypes = [u64, u64, i32, i32, vp, vp]
        L.synth_f32_to_bf16.argtypes = [vp, u64, vp]
        for f in ("synth_words", "synth_codes", "synth_scale_bias", "synth_normal_f32",
                  "synth_zipf_gumbel_logits", "synth_f32_to_bf16"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def key(seed: int, kind: int, layer: int, slot: int) -> int:
    return int(lib().synth_key(seed, kind, layer, slot))


def words(k: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    lib().synth_words(k, first, n, _p(out))
    return out


def codes(k: int, bits: int, n: int, first: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint8)
    lib().synth_codes(k, bits, first, n, _p(out))
    return out


def normal_f32(k: int, n: int, mean: float = 0.0, std: float = 1.0, first: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_f32(k, mean, std, first, n, _p(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().synth_f32_to_bf16(_p(x), x.size, _p(out))
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """Shape and value distributions of one MoE layer."""

    hidden: int = 4096
    inter: int = 1024
    n_experts: int = 512
    top_k: int = 4
    bits: int = 4          # routed experts
    shared_bits: int = 4   # the shared expert
    group: int = 64
    eps: float = 1e-6
    seed: int = 0

    def scale_range(self, bits: int) -> tuple[float, float]:
        return (0.005, 0.02) if bits == 4 else (0.02, 0.08)

    @property
    def bias_sigma(self) -> float:
        return 1e-3

    def expert_bits(self, slot: int) -> int:
        return self.shared_bits if slot == self.n_experts else self.bits


TINY = Workload(hidden=256, inter=128, n_experts=16)
LAYER = Workload()
LAYER_INT2 = Workload(bits=2)


@dataclass
class ExpertLogical:
    """Logical (unpacked) tensors of one expert; matrices in order gate, up, down.

    q      uint8 [3 * inter * hidden]: gate [inter][hidden], up [inter][hidden],
           down [hidden][inter], row-major, one code per byte.
    scale  uint16 (bf16 bits) [3 * inter * hidden / group], row-major per matrix.
    bias   uint16 (bf16 bits), same layout as scale.
    """

    bits: int
    q: np.ndarray
    scale: np.ndarray
    bias: np.ndarray

    def matrices(self, wl: Workload):
        H, I, G = wl.hidden, wl.inter, wl.group
        n = H * I
        ng = n // G
        shapes = [(I, H), (I, H), (H, I)]
        out = []
        for m, (r, c) in enumerate(shapes):
            out.append((self.q[m * n:(m + 1) * n].reshape(r, c),
                        self.scale[m * ng:(m + 1) * ng].reshape(r, c // G),
                        self.bias[m * ng:(m + 1) * ng].reshape(r, c // G)))
        return out


def expert(wl: Workload, layer: int, slot: int, out: ExpertLogical | None = None) -> ExpertLogical:
    """Generate expert `slot` (0..E-1 routed, E = shared) of `layer`."""
    L = lib()
    bits = wl.expert_bits(slot)
    n = wl.hidden * wl.inter
    ng = n // wl.group
    if out is None:
        out = ExpertLogical(bits, np.empty(3 * n, np.uint8), np.empty(3 * ng, np.uint16),
                            np.empty(3 * ng, np.uint16))
    lo, hi = wl.scale_range(bits)
    for m in range(3):
        kc = key(wl.seed, K_CODES[m], layer, slot)
        L.synth_codes(kc, bits, 0, n, ctypes.c_void_p(out.q.ctypes.data + m * n))
        ks = key(wl.seed, K_SCALE[m], layer, slot)
        kb = key(wl.seed, K_BIAS[m], layer, slot)
        L.synth_scale_bias(ks, kb, bits, lo, hi, wl.bias_sigma, 0, ng,
                           ctypes.c_void_p(out.scale.ctypes.data + 2 * m * ng),
                           ctypes.c_void_p(out.bias.ctypes.data + 2 * m * ng))
    return out


def experts(wl: Workload, layer: int, slots, threads: int | None = None) -> list[ExpertLogical]:
    slots = list(slots)
    threads = threads or min(len(slots), os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        return list(ex.map(lambda s: expert(wl, layer, s), slots))


def router(wl: Workload, layer: int) -> np.ndarray:
    """Router weights, fp32 [n_experts][hidden] ~ N(0, 0.02)."""
    return normal_f32(key(wl.seed, K_ROUTER, layer, 0), wl.n_experts * wl.hidden, 0.0, 0.02).reshape(
        wl.n_experts, wl.hidden)


def shared_gate(wl: Workload, layer: int) -> np.ndarray:
    """Shared-expert gate vector, fp32 [hidden] ~ N(0, 0.02)."""
    return normal_f32(key(wl.seed, K_SHARED_GATE, layer, 0), wl.hidden, 0.0, 0.02)


def norm_weight(wl: Workload, layer: int) -> np.ndarray:
    """RMSNorm weight, fp32 [hidden] ~ 1 + N(0, 0.1)."""
    return normal_f32(key(wl.seed, K_NORM, layer, 0), wl.hidden, 1.0, 0.1)


def tokens(wl: Workload, n_tokens: int, stream: int = 0, first_token: int = 0) -> np.ndarray:
    """Token inputs x ~ N(0, 1) fp32 [n_tokens][hidden]; `stream` separates steps."""
    out = np.empty((n_tokens, wl.hidden), np.float32)
    for t in range(n_tokens):
        out[t] = normal_f32(key(wl.seed, K_X, stream, first_token + t), wl.hidden)
    return out


def zipf_gumbel_logits(wl: Workload, step: int, n_tokens: int) -> tuple[np.ndarray, np.ndarray]:
    """Router logits of one batched step: Zipf(1) popularity + Gumbel noise.

    Returns (logits fp32 [n_tokens][n_experts], rank_to_id int32 [n_experts]).
    The popularity permutation is fixed per seed; the noise is fresh per step.
    """
    logits = np.empty((n_tokens, wl.n_experts), np.float32)
    r2i = np.empty(wl.n_experts, np.int32)
    lib().synth_zipf_gumbel_logits(key(wl.seed, K_ZIPF_PERM, 0, 0), key(wl.seed, K_GUMBEL, step, 0),
                                   n_tokens, wl.n_experts, _p(logits), _p(r2i))
    return logits, r2i
