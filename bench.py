"""Benchmark: MoE-layer expert forwards per second at batch 1 on B200.

Workload: one 4-bit MoE layer of hidden 4096, expert intermediate 1024, 512
routed experts (top-4, softmax renormalised over the selected) plus one
shared expert, group-64 affine codes with bf16 scale/bias (6.75 MiB per
expert, 3.62 GB per layer).  `--layers` (default 20) copies of that layer are
resident in HBM (72.5 GB) and a token is carried through them as a stack, so
that every step reads a new router, a new shared expert and the 4 routed
experts the token picks: one step = one layer forward of one token, and the
same weights come back only after 19 other layers (> 800 MB of other reads,
well above the 126 MB L2).  All inputs are synthetic and seeded.

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank runs its own
replica (the path has no exchange step) and the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer expert fwd/s at batch 1; weight-stream HBM GB/s vs B200 peak"
UNIT = "layer_fwd/s"
DTYPE = ("int4 codes x 24-bit block floating-point activations (one power-of-two step per 64 inputs, "
         "the fp32 significand at the group maximum), exact int32 group dots, fp32 epilogue and accumulation")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=20, help="resident layer copies (L2 rotation)")
    ap.add_argument("--experts", type=int, default=512, help="routed experts per layer (fewer only to profile small)")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the oracle CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the batched and 2-bit chain measurements")
    ap.add_argument("--int2-layers", type=int, default=20, help="resident 2-bit layers of the 2-bit chain (0: skip)")
    return ap.parse_args()


def batched_measure(fm, synth, np, torch, lw, wl, stream, steps=50, warmup=5, T=64):
    """64 tokens per step through one layer, top-4 drawn from Zipf(1) expert
    popularity (fresh Gumbel-top-k logits every step, given as router
    logits): tokens/s and the expert bytes the steps touch."""
    logits = [torch.from_numpy(synth.zipf_gumbel_logits(wl, s, T)[0]).cuda() for s in range(steps)]
    hot, tc_min = [], fm.fmoe_tc_min_tokens()
    for lg in logits:
        ids = torch.topk(lg, wl.top_k, dim=1).indices.cpu().numpy()
        cnt = np.bincount(ids.ravel(), minlength=wl.n_experts)
        hot.append(((cnt > 0).sum(), (cnt >= tc_min).sum()))
    x = torch.from_numpy(synth.tokens(wl, T, stream=900)).cuda()
    h, xn = x.clone(), x.clone()
    ws = fm.alloc_workspace(lw.desc, T)
    with torch.cuda.stream(stream):
        for s in range(warmup):
            fm.fmoe_layer_forward_logits(lw, logits[s % steps], h, xn, ws, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for s in range(steps):
            fm.fmoe_layer_forward_logits(lw, logits[s], h, xn, ws, stream=stream)
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    rec = lw.desc.record_bytes()
    distinct = float(np.mean([d for d, _ in hot]))
    bytes_step = (distinct + 1) * rec  # routed experts touched + the shared expert
    return {"workload": f"moe_layer_int4_batch{T}_zipf: {T} tokens per step through one 512-expert layer, Zipf(1) "
                        f"top-4 routing (fresh Gumbel-top-k logits each step, given), {steps} steps",
            "tokens_per_s": T * steps / (ms / 1e3), "ms_per_step": ms / steps,
            "distinct_experts_per_step": distinct, "tensor_core_experts_per_step": float(np.mean([t for _, t in hot])) + 1,
            "expert_weight_gbs": bytes_step * steps / (ms / 1e3) / 1e9,
            "timing": "CUDA events on the launching stream, 50 consecutive steps"}


def small_batch_measure(fm, synth, torch, layers, wl, stream, Ts=(2, 4, 8), rotations=20):
    """T tokens (2-15: a small decode batch or a speculative-verify step)
    carried through the resident layer stack, routed by the layers' own
    routers: one CUDA graph replay per rotation of the stack, CUDA events
    around `rotations` replays.  Per T: microseconds per layer and token-
    layers per second."""
    out = {}
    L = len(layers)
    for T in Ts:
        x = torch.from_numpy(synth.tokens(wl, T, stream=950 + T)).cuda()
        h, xn = x.clone(), x.clone()
        ws = fm.alloc_workspace(layers[0].desc, T)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            fm.fmoe_stack_forward(layers, h, xn, ws, stream=stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                fm.fmoe_stack_forward(layers, h, xn, ws, stream=stream)
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(rotations):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (rotations * L)
        out[str(T)] = {"us_per_layer": us, "layer_fwd_per_s": 1e6 / us, "token_layers_per_s": T * 1e6 / us}
        del g
    return {"workload": f"moe_stack_int4_small_batch: T tokens through the {L} resident int4 layers (routed by "
                        f"their routers), {rotations} graph replays of the stack per T",
            "by_T": out}


def cache_measure(fm, synth, np, torch, layers, wl, stream, n_layers=4, slot_counts=(64, 256, 1024), tokens=50):
    """Decode (T = 1) through `n_layers` layers whose routed experts live in
    pinned host memory, with a device cache of `slots` records shared by the
    layers (least recently used first); routing from Zipf(1)-popularity
    Gumbel-top-k logits per layer and token.  Per cache size: layer steps/s,
    hit rate, host-to-device expert GB/s."""
    n_layers = min(n_layers, len(layers))
    host = [layers[l].experts.cpu().pin_memory() for l in range(n_layers)]
    logits = [[torch.from_numpy(synth.zipf_gumbel_logits(wl, 1000 * l + t, 1)[0]).cuda() for l in range(n_layers)]
              for t in range(tokens)]
    x = torch.from_numpy(synth.tokens(wl, 1, stream=960)).cuda()
    ws = fm.alloc_workspace(layers[0].desc, 1)
    out = {}
    for slots in slot_counts:
        cache = fm.ExpertCache(layers[0].desc, host, n_slots=slots, max_tokens=1)
        h, xn = x.clone(), x.clone()
        with torch.cuda.stream(stream):
            for t in range(5):  # warm the cache
                for l in range(n_layers):
                    cache.forward(l, layers[l], h, xn, ws, logits=logits[t][l], stream=stream)
        torch.cuda.synchronize()
        h0, m0, b0 = cache.stats()
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            for t in range(tokens):
                for l in range(n_layers):
                    cache.forward(l, layers[l], h, xn, ws, logits=logits[t][l], stream=stream)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
        h1, m1, b1 = cache.stats()
        steps = tokens * n_layers
        out[str(slots)] = {"layer_steps_per_s": steps / dt, "hit_rate": (h1 - h0) / max(1, (h1 - h0) + (m1 - m0)),
                           "h2d_gbs": (b1 - b0) / dt / 1e9, "slots_gb": slots * layers[0].desc.record_bytes() / 1e9}
        cache.close()
        del cache
        torch.cuda.empty_cache()
    del host
    return {"workload": f"moe_decode_host_tier: {n_layers} int4 layers' routed experts in pinned host memory, device "
                        f"cache of N records shared by the layers (LRU), Zipf(1) routing, {tokens} tokens",
            "timing": "host wall clock around the steps (each step synchronises to read its routing)",
            "by_slots": out}


def quantiser_measure(fm, torch, stream, experts=16, reps=10, H=4096, I=1024):
    """The device quantiser (fp32 weights -> int4 codes + bf16 scale/bias) on
    `experts` experts' worth of fp32 weights (3 H I each): GB/s of fp32
    weights read (bytes moved: 4 in, 1 code + 4/64 scale-bias out per
    weight)."""
    n = experts * 3 * H * I
    g = torch.Generator(device="cuda").manual_seed(5)
    w = torch.randn(n, device="cuda", generator=g) * 0.02
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n // 64, dtype=torch.int16, device="cuda")
    bi = torch.empty(n // 64, dtype=torch.int16, device="cuda")
    with torch.cuda.stream(stream):
        for _ in range(2):
            fm.fmoe_quantize_groups(w, 4, q, sc, bi, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            fm.fmoe_quantize_groups(w, 4, q, sc, bi, stream=stream)
        e1.record(stream)
    e1.synchronize()
    s = e0.elapsed_time(e1) / 1e3 / reps
    moved = n * 4 + n + (n // 64) * 4
    del w, q, sc, bi
    return {"workload": f"quantise {experts} experts' fp32 weights (hidden {H}, inter {I}) to int4 + bf16 scale/bias",
            "ms": s * 1e3, "weights_per_s": n / s, "gbs_moved": moved / s / 1e9}


def int2_chain_measure(fm, synth, torch, stream, layers=20, steps=2000, warmup=100):
    """The 2-bit variant of the layer stack (routed experts 2-bit, shared
    expert 4-bit), one token carried through all layers: layers/s."""
    wl = synth.LAYER_INT2
    scratch = {}
    lws = [synth_device_upload(synth, wl, l, scratch) for l in range(layers)]
    del scratch
    torch.cuda.empty_cache()
    x = torch.from_numpy(synth.tokens(wl, 1, stream=901)).cuda()
    h, xn = x.clone(), x.clone()
    ws = fm.alloc_workspace(lws[0].desc, 1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fm.fmoe_stack_forward(lws, h, xn, ws, stream=stream)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fm.fmoe_stack_forward(lws, h, xn, ws, stream=stream)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup // layers)):
            g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, steps // layers)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n):
            g.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    d = lws[0].desc
    layer_bytes = 4 * d.record_bytes() + d.record_bytes(shared=True) + wl.n_experts * wl.hidden * 4 + 2 * wl.hidden * 4
    per_layer_s = ms / 1e3 / (n * layers)
    del g
    return {"workload": f"moe_stack_int2_batch1: {layers} resident layers, 2-bit routed experts (3.75 MiB), 4-bit "
                        f"shared expert, one token carried through the stack",
            "layer_fwd_per_s": 1 / per_layer_s, "tokens_per_s": 1 / per_layer_s / layers,
            "layer_gbs": layer_bytes / per_layer_s / 1e9, "bytes_per_layer": layer_bytes}


def synth_device_upload(synth, wl, layer, scratch):
    from synth.device import upload_layer
    return upload_layer(wl, layer, scratch=scratch)


def workload_config(layers: int, experts: int = 512) -> dict:
    return {
        "workload": f"moe_layer_int4_batch1: hidden 4096, expert inter 1024, {experts} experts top-4 + 1 shared, "
                    f"group-64 int4 bf16 scale/bias, {layers} resident layer copies chained (one step = one layer of one token)",
        "hidden": 4096, "inter": 1024, "experts": experts, "top_k": 4, "shared_experts": 1, "bits": 4, "group": 64,
        "batch": 1, "layer_copies": layers,
        "l2": f"inputs larger than L2: rotation over {layers} resident layers ({layers * 43.8:.0f} MB of weights per rotation)",
    }


# DRAM bytes (read + write) of one full-size int4 layer of fused_stack_kernel,
# from an ncu capture (profiles/fused_stack_kernel_int4_batch1.md), valid for
# the kernel sources whose digest is given; any later change to them voids it.
TRAFFIC_PER_LAYER = {"sources_sha256_16": "9aba729bf237347f", "bytes": 43_996_672}
TRAFFIC_SOURCES = ("fmoe_fused.cuh", "fmoe_device.cuh", "fmoe_layout.h")  # the kernel's sources


def measured_traffic(layers: int):
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "quantized_expert_gemv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != TRAFFIC_PER_LAYER["sources_sha256_16"]:
        return None
    return TRAFFIC_PER_LAYER["bytes"] * layers


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period: float = 0.01):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                import torch
                p = torch.cuda.get_device_properties(device_index)
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._sample()

            def loop():
                while not self._stop.wait(self.period):
                    self._sample()
            self._t = threading.Thread(target=loop, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ distributed --
def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time (every rank takes part; `device` is where the
    reduction runs: the rank's GPU under NCCL, "cpu" under gloo)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas that each processed
    units_per_rank units, timed by the slowest rank."""
    return world * units_per_rank / (ms_max / 1e3)


# ----------------------------------------------------------- CPU baseline --
def oracle_layer_steps(max_steps: int, seconds: float, layers: int, wl=None):
    """Times the fp64 oracle, as it stands, on the host (one thread or, after
    oracle.set_threads, the OpenMP timing build): successive
    single-token layer forwards of the benchmark workload (or `wl`) through
    the layer stack, until `max_steps` are done or `seconds` of oracle time
    are spent.  The selected experts are regenerated on demand; generation is
    not timed.  Returns (steps done, seconds spent in the oracle)."""
    import numpy as np
    import oracle
    import synth
    wl = wl or synth.LAYER
    done, spent = 0, 0.0
    cache = {}
    while done < max_steps and spent < seconds:
        l = done % layers
        if l not in cache:
            cache[l] = oracle.LayerWeights(synth.router(wl, l), synth.shared_gate(wl, l), synth.norm_weight(wl, l), {})
        lw = cache[l]
        x = synth.tokens(wl, 1, stream=1000 + done)[0].astype(np.float64)
        lg, _ = oracle.gemv_f32(lw.w_router, x)
        ids, _, _ = oracle.topk_softmax(lg, wl.top_k)
        lw.experts = {int(s): synth.expert(wl, l, int(s)) for s in list(ids) + [wl.n_experts]}
        t0 = time.perf_counter()
        oracle.layer_token(wl, lw, x, x)
        spent += time.perf_counter() - t0
        done += 1
    return done, spent


def oracle_batched_tokens(n_tokens: int, T: int = 64):
    """Times the fp64 oracle on the first n_tokens tokens of the 64-token
    Zipf-routed step of the batched measurement (the same routing draw,
    given logits): per token the layer with its selected experts, which the
    oracle computes token by token.  Expert generation is not timed.
    Returns (tokens done, seconds spent in the oracle)."""
    import numpy as np
    import oracle
    import synth
    wl = synth.LAYER
    lg = synth.zipf_gumbel_logits(wl, 0, T)[0]
    xs = synth.tokens(wl, T, stream=900)
    lw = oracle.LayerWeights(synth.router(wl, 0), synth.shared_gate(wl, 0), synth.norm_weight(wl, 0),
                             {wl.n_experts: synth.expert(wl, 0, wl.n_experts)})
    spent = 0.0
    for t in range(n_tokens):
        ids, _, _ = oracle.topk_softmax(lg[t].astype(np.float64), wl.top_k)
        for e in ids:
            if int(e) not in lw.experts:
                lw.experts[int(e)] = synth.expert(wl, 0, int(e))
        x = xs[t].astype(np.float64)
        t0 = time.perf_counter()
        oracle.layer_token(wl, lw, x, x, logits_in=lg[t])
        spent += time.perf_counter() - t0
    return n_tokens, spent


def host_cores() -> int:
    """Cores this process may run on (the affinity mask, not the machine)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(seconds: float, layers: int) -> dict:
    """The oracle on all the host cores this process may use (OpenMP over
    the output rows of its products; the same values as one thread), and on
    one thread; each a bounded sample of `seconds` / 2."""
    import oracle
    cores = host_cores()
    oracle.set_threads(cores)
    done, spent = oracle_layer_steps(10 ** 6, seconds / 2, layers)
    # the other workloads, on all cores, small bounded samples
    import synth
    d2, s2 = oracle_layer_steps(10 ** 6, min(3.0, seconds / 5), layers, wl=synth.LAYER_INT2)
    nb, sb = oracle_batched_tokens(8)
    oracle.set_threads(1)
    done1, spent1 = oracle_layer_steps(10 ** 6, seconds / 2, layers)
    return {"value": done / spent, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} single-token layer forwards of the benchmark workload (fp64 C oracle, OpenMP over "
                      f"output rows on {cores} cores; expert generation excluded), {spent:.1f} s",
            "single_thread": {"value": done1 / spent1, "unit": UNIT, "cores": 1,
                              "sample": f"{done1} layer forwards on one thread, {spent1:.1f} s"},
            "int4_chain_tokens_per_s": done / spent / layers,
            "int2_chain": {"layer_fwd_per_s": d2 / s2, "tokens_per_s": d2 / s2 / layers, "cores": cores,
                           "sample": f"{d2} layer forwards of 2-bit routed / 4-bit shared layers, {s2:.1f} s"},
            "batched": {"tokens_per_s": nb / sb, "ms_per_64_token_step": 64 * sb / nb * 1e3, "cores": cores,
                        "sample": f"the first {nb} tokens of the 64-token Zipf step (given logits), "
                                  f"{sb:.1f} s; the oracle computes token by token"}}


def run_reference(args):
    """The oracle as the reference arm: rank 0 alone times it on the host
    cores (OpenMP over output rows on every core of its affinity mask;
    bounded sample: at most `steps` layer forwards or ~150 s)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cores = oracle.set_threads(host_cores())
    oracle_layer_steps(min(args.warmup, 1), 1e9, args.layers)
    done, spent = oracle_layer_steps(max(1, args.steps), 150.0, args.layers)
    value = done / spent
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": done,
            "warmup": args.warmup, "ms_per_step": 1e3 * spent / done, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(args.layers),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{done} single-token layer forwards (fp64 C oracle, OpenMP over output rows "
                                       f"on {cores} cores; expert generation excluded), {spent:.1f} s of "
                                       f"{max(1, args.steps)} requested steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours --
def run_ours(args):
    import numpy as np
    import torch

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    import quantized_expert_gemv_b200 as fm
    import synth
    from synth.device import upload_layer

    wl = synth.LAYER if args.experts == 512 else synth.Workload(n_experts=args.experts)
    L = args.layers
    scratch = {}
    layers = [upload_layer(wl, l, scratch=scratch) for l in range(L)]
    del scratch
    torch.cuda.empty_cache()
    desc = layers[0].desc
    H = wl.hidden
    ws = fm.alloc_workspace(desc, 1)
    x0 = synth.tokens(wl, 1, stream=7 + rank)
    h = torch.from_numpy(x0).cuda()
    xn = h.clone()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    # graphs: one per layer copy, and one for a whole rotation
    graphs = []
    with torch.cuda.stream(stream):
        for l in range(L):  # eager warm-up of every layer once
            fm.fmoe_layer_forward(layers[l], h, xn, ws, stream=stream)
        stream.synchronize()
        for l in range(L):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fm.fmoe_layer_forward(layers[l], h, xn, ws, stream=stream)
            graphs.append(g)
        g_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_all, stream=stream):
            fm.fmoe_stack_forward(layers, h, xn, ws, stream=stream)
    torch.cuda.synchronize()

    def run_steps(n):
        i = 0
        while i + L <= n:
            g_all.replay()
            i += L
        while i < n:
            graphs[i % L].replay()
            i += 1

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
        for _ in range(3):  # the timed region replays the whole-rotation graph: warm it too
            g_all.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world)
    st = fm.fmoe_read_status(clear=True)
    if st:
        raise RuntimeError(f"device status word {st:#x} after the timed region")

    per_step_s = ms_max / 1e3 / args.steps
    value = job_rate(args.steps, world, ms_max)
    rec = desc.record_bytes()
    expert_bytes = (wl.top_k + 1) * rec
    layer_bytes = expert_bytes + wl.n_experts * H * 4 + 2 * H * 4
    peak, peak_kind = measured_peak()
    achieved = layer_bytes / per_step_s / 1e9
    n_full = args.steps // L
    launches = n_full + (args.steps - n_full * L)
    roofline = {"bound": "hbm",
                "kernel": f"fused_stack_kernel: whole layers (router, top-k, gate/up+SwiGLU, down, combine+RMSNorm), "
                          f"{L} layers per launch",
                "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": measured_traffic(L) if wl.n_experts == 512 else None,
                "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one full-size layer launch, "
                                "times the layers per launch (per-layer traffic is additive)",
                "bytes_per_layer": layer_bytes, "layers_per_launch": L,
                "timing": "CUDA events on the launching stream around the timed replays"}

    # ---- end to end through the C ABI with host buffers (eager calls) ----
    # A plain C decode loop: per call, one token's [2, 1, H] block (h and its
    # normed copy xn) is copied from pinned host memory to the device, the L
    # resident layers run, and h', xn' are copied back (fmoe_stack_forward_host).
    # One call = L steps.
    K2 = args.e2e_steps or max(min(args.steps, 2000), 10 * L)
    calls = max(1, K2 // L)
    K2 = calls * L
    xs = synth.tokens(wl, min(calls, 64), stream=500 + rank)
    nb = xs.shape[0]
    hx_in = torch.from_numpy(np.ascontiguousarray(np.stack([xs, xs], axis=1)[:, :, None, :])).pin_memory()
    hx_out = torch.empty((nb, 2, 1, H), dtype=torch.float32).pin_memory()
    hx = torch.empty((2, 1, H), dtype=torch.float32, device="cuda")

    def e2e_calls(n):
        for i in range(n):
            j = i % nb
            fm.fmoe_stack_forward_host(layers, hx_in[j], hx_out[j], hx, ws, stream=stream)

    with torch.cuda.stream(stream):
        e2e_calls(min(5, calls))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        e2e_calls(calls)
        e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e = {"value": job_rate(K2, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": 2 * H * 4 / L,
           "d2h_bytes_per_step": 2 * H * 4 / L, "steps": K2, "calls": calls,
           "how": f"per call (= {L} steps): fmoe_stack_forward_host, one eager C-ABI call: a pinned host [2, H] block "
                  f"(h, xn) -> device, the {L} resident layers, h', xn' -> pinned host ({2 * H * 4} bytes each way "
                  f"per call)"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
            "data": "synthetic (seeded generator, random-init weights of the layer shape)",
            "config": workload_config(L, wl.n_experts),
            "expert_weight_gbs": expert_bytes / per_step_s / 1e9,
            "layer_gbs": achieved,
            "pct_of_8tbs_expert_bytes": 100 * expert_bytes / per_step_s / 8e12,
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk.summary()}
    line["tokens_per_s"] = value / L  # one token through the L-layer stack
    # the further measurements run on a single-GPU run only (under torchrun
    # every rank would repeat them, pinning host memory per rank)
    if not args.no_extra and wl.n_experts == 512 and world == 1:
        line["batched"] = batched_measure(fm, synth, np, torch, layers[0], wl, stream)
        line["small_batch"] = small_batch_measure(fm, synth, torch, layers, wl, stream)
        line["quantiser"] = quantiser_measure(fm, torch, stream)
        line["host_tier"] = cache_measure(fm, synth, np, torch, layers, wl, stream)
        del layers, graphs, g_all
        graphs = g_all = None
        torch.cuda.empty_cache()
        if args.int2_layers > 0:
            line["int2_chain"] = int2_chain_measure(fm, synth, torch, stream, layers=args.int2_layers)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds, L)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world)
    del graphs, g_all
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
