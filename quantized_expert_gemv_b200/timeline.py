"""Per-phase timeline of the persistent layer-stack kernel.

Builds the library with FMOE_TIMELINE (timer reads at the kernel's phase
boundaries, see fmoe_fused.cuh) as libfmoe_timeline.so beside the product
library, runs a stack of resident layers through fmoe_stack_forward from
that build, and prints, per phase, the minimum / median / maximum over the
CTAs of the time (us) from the earliest CTA's start of the recorded layer.
The product library carries no timer reads.

    python -m quantized_expert_gemv_b200.timeline [--layers 20] [--record 5]
        [--inter 1024] [--experts 512]
"""
from __future__ import annotations

import argparse
import ctypes
import os

import numpy as np

from . import build as _build

POINTS = {
    0: "layer start",
    1: "A: every CTA's h' visible",
    2: "A: xn = h' r w computed",
    3: "A: xn staged",
    4: "A: router rows in shared memory",
    5: "A: router dot products",
    6: "A: logits published",
    **{7 + p: f"gu: block {p} bytes landed" for p in range(5)},
    **{12 + p: f"gu: block {p} SwiGLU outputs staged" for p in range(5)},
    17: "dn: every CTA's logits counted",
    18: "dn: warp top-k done",
    19: "dn: top-k merged, softmax",
    20: "dn: routed copies issued",
    **{21 + p: f"dn: block {p} ready" for p in range(5)},
    **{26 + p: f"dn: block {p} down products done" for p in range(5)},
    31: "F: partial output stored",
    32: "F: partial published",
    33: "G: every CTA's partial visible",
    34: "G: slice sums",
    35: "G: h' published",
}
N_POINTS = 48
MAX_CTAS = 160


def build_timeline_lib(force: bool = False) -> str:
    out = os.path.join(_build.PKG, "libfmoe_timeline.so")
    return _build.build(force=force, extra_flags=["-DFMOE_TIMELINE"], out=out)


def run(layers: int = 20, record: int = 5, inter: int = 1024, experts: int = 512, repeats: int = 5):
    import torch

    import quantized_expert_gemv_b200 as fm
    import synth
    from synth.device import upload_layer

    lib = ctypes.CDLL(build_timeline_lib())
    lib.fmoe_stack_forward.argtypes = [ctypes.POINTER(fm.fmoe_layer_weights), ctypes.c_int, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]
    lib.fmoe_timeline_layer.argtypes = [ctypes.c_int]
    lib.fmoe_timeline_read.argtypes = [ctypes.c_void_p]
    wl = synth.LAYER if (inter, experts) == (1024, 512) else synth.Workload(inter=inter, n_experts=experts)
    scratch = {}
    lws = [upload_layer(wl, l, scratch=scratch) for l in range(layers)]
    del scratch
    arr = (fm.fmoe_layer_weights * layers)(*[lw.c() for lw in lws])
    ws = fm.alloc_workspace(lws[0].desc, 1)
    x = torch.from_numpy(synth.tokens(wl, 1, stream=3)).cuda()
    h, xn = x.clone(), x.clone()
    st = torch.cuda.current_stream().cuda_stream
    assert lib.fmoe_timeline_layer(record) == 0

    def launch():
        rc = lib.fmoe_stack_forward(arr, layers, ctypes.c_void_p(h.data_ptr()), ctypes.c_void_p(xn.data_ptr()), 1,
                                    ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(st))
        assert rc == 0, rc

    for _ in range(repeats):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(repeats):
        launch()
    e1.record()
    torch.cuda.synchronize()
    per_layer = e0.elapsed_time(e1) * 1e3 / (repeats * layers)
    ts = np.zeros((MAX_CTAS, N_POINTS), np.uint64)
    assert lib.fmoe_timeline_read(ctypes.c_void_p(ts.ctypes.data)) == 0
    n = torch.cuda.get_device_properties(0).multi_processor_count
    t = ts[:min(n, MAX_CTAS)].astype(np.int64)
    t0 = t[:, 0][t[:, 0] > 0].min()
    rows = []
    for i, name in POINTS.items():
        v = t[:, i][t[:, i] > 0]
        if len(v):
            r = (v - t0) / 1e3
            rows.append((float(np.median(r)), name, float(r.min()), float(r.max()), len(v)))
    print(f"{layers} layers per launch, layer {record} recorded: {per_layer:.2f} us per layer (with timer reads)")
    print(f"{'phase':42s} {'min':>7s} {'median':>7s} {'max':>7s}  CTAs")
    for med, name, lo, hi, cnt in sorted(rows):
        print(f"{name:42s} {lo:7.2f} {med:7.2f} {hi:7.2f}  {cnt}")
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=20)
    ap.add_argument("--record", type=int, default=5)
    ap.add_argument("--inter", type=int, default=1024)
    ap.add_argument("--experts", type=int, default=512)
    a = ap.parse_args()
    run(a.layers, a.record, a.inter, a.experts)


if __name__ == "__main__":
    main()
