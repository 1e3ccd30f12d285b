"""GPU parity: every C-ABI entry point against the fp64 CPU oracle.

Inputs come from the seeded generator (synth); the oracle computes on the
logical layout, the device on the packed layout through libfmoe.  Router
top-k is compared bit-exactly on the device's own fp32 logits; every float
output within |d - v| <= 1e-3 S + 1e-5 and relative L2 <= 2e-3 (tests/parity.py).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import layer_desc, upload_layer
from tests.parity import check, pmap

pytestmark = pytest.mark.gpu

fm = pytest.importorskip("quantized_expert_gemv_b200")

TINY2 = synth.Workload(hidden=256, inter=128, n_experts=16, bits=2)
# small shapes the persistent fused kernel accepts (inter a multiple of 256)
SMALL = synth.Workload(hidden=256, inter=256, n_experts=16)
SMALL2 = synth.Workload(hidden=256, inter=256, n_experts=16, bits=2)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fm.fmoe_read_status(clear=True)
    yield
    torch.cuda.synchronize()


def oracle_layer(wl, layer, slots=None):
    lw = oracle.LayerWeights(synth.router(wl, layer), synth.shared_gate(wl, layer), synth.norm_weight(wl, layer), {})
    slots = range(wl.n_experts + 1) if slots is None else slots
    for s, ex in zip(slots, synth.experts(wl, layer, slots)):
        lw.experts[int(s)] = ex
    return lw


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


_layers = {}


def device_layer(wl, layer=0):
    key = (wl, layer)
    if key not in _layers:
        _layers[key] = upload_layer(wl, layer)
    return _layers[key]


def fused_on():
    prev = fm.fmoe_set_fused(True)
    fm.fmoe_set_fused(prev)
    return prev


def check_layer_token(wl, lw_o, ws, desc, T, t, h_in, xn_in, h_out, xn_out, label, logits_given=False):
    """Teacher-forced check of token t of one layer step: routing on the
    device's fp32 logits (the router product is checked too unless the
    logits were given), then each expert's SwiGLU outputs a, the expert
    outputs y (left in the workspace by the one-kernel-per-step path only;
    the persistent kernel sums them on the fly), h' and xn' against the
    oracle."""
    fused = T <= fm.fmoe_fused_max_tokens() and not logits_given and fused_on() and fm.fmoe_fused_supported(desc)
    v = {name: host(fm.workspace_view(ws, desc, T, which))[t]
         for name, which in (("logits", fm.WS_LOGITS), ("ids", fm.WS_IDS), ("p", fm.WS_WEIGHTS),
                             ("gamma", fm.WS_GAMMA), ("a", fm.WS_A), ("y", fm.WS_Y))}
    if fused:
        del v["y"]
    return check_layer_values(wl, lw_o, v, h_in, xn_in, h_out, xn_out, label, logits_given)


def check_layer_values(wl, lw_o, v, h_in, xn_in, h_out, xn_out, label, logits_given=False):
    """check_layer_token on the intermediates v (logits, ids, p, gamma, a and,
    when present, y) of one token's layer step."""
    layer = getattr(lw_o, "layer", 0)
    # a private copy of the layer: experts generated for this check are dropped with it
    lw_o = oracle.LayerWeights(lw_o.w_router, lw_o.w_shared_gate, lw_o.norm_w, dict(lw_o.experts))
    lg_d, ids_d, p_d, a_d, gamma_d = v["logits"], v["ids"], v["p"], v["a"], v["gamma"]
    if not logits_given:
        lg_o, S_l = oracle.gemv_f32(lw_o.w_router, xn_in.astype(np.float64))
        check(lg_d, lg_o, S_l, f"{label} logits")
    ref = oracle.layer_token(wl, lw_o, h_in.astype(np.float64), xn_in.astype(np.float64), logits_in=lg_d,
                             expert_fn=lambda s: synth.expert(wl, layer, s))
    assert ref["ids"].tolist() == ids_d.tolist(), f"{label} ids {ids_d} vs oracle {ref['ids']}"
    check(p_d, ref["p"], ref["p"], f"{label} gate weights")
    # gamma is a scalar: checked per element (relative L2 is taken over vector
    # outputs; a strongly negative gate logit gives an fp64 gamma far below
    # the fp32 range, which the device stores as 0)
    check(gamma_d, ref["gamma"], ref["gamma"] + ref["S_gamma"], f"{label} gamma", rel_l2=False)
    for j, slot in enumerate(list(ids_d) + [wl.n_experts]):
        e = oracle.expert_ffn(lw_o.experts[int(slot)], wl.hidden, wl.inter, wl.group, xn_in)
        check(a_d[j], e["a"], e["S_a"], f"{label} a[{j}]")
    if "y" in v:
        check(v["y"], ref["y"], ref["S_y"], f"{label} y")
    check(h_out, ref["h"], ref["S_h"], f"{label} h'")
    check(xn_out, ref["xn"], ref["S_xn"], f"{label} xn'")
    return ref


TRACE_SECTIONS = (("xn_in", fm.TRACE_XN_IN), ("logits", fm.TRACE_LOGITS), ("ids", fm.TRACE_IDS),
                  ("p", fm.TRACE_WEIGHTS), ("gamma", fm.TRACE_GAMMA), ("a", fm.TRACE_A), ("h", fm.TRACE_H_OUT))


def traced_stack_check(wl, lws, los, x, label):
    """x [T][H] through the stack (h = xn = x) with a trace; every layer of
    every token checked teacher-forced on the values the launch recorded.
    Returns the final h', xn'."""
    desc = lws[0].desc
    T, L = len(x), len(lws)
    ws = fm.alloc_workspace(desc, T)
    tr = fm.alloc_trace(desc, T, L)
    h, xn = dev(x), dev(x)
    fm.fmoe_stack_forward(lws, h, xn, ws, trace=tr)
    rec = [{name: host(fm.trace_view(tr, desc, T, l, which)) for name, which in TRACE_SECTIONS} for l in range(L)]
    h_fin, xn_fin = host(h), host(xn)
    assert np.array_equal(rec[-1]["h"], h_fin)
    jobs = [(l, t) for l in range(L) for t in range(T)]

    def job(j):
        l, t = jobs[j]
        h_in = x[t] if l == 0 else rec[l - 1]["h"][t]
        xn_out = rec[l + 1]["xn_in"][t] if l + 1 < L else xn_fin[t]
        v = {name: rec[l][name][t] for name in ("logits", "ids", "p", "gamma", "a")}
        check_layer_values(wl, los[l], v, h_in, rec[l]["xn_in"][t], rec[l]["h"][t], xn_out,
                           f"{label} stack layer {l} t={t}")

    pmap(job, range(len(jobs)))
    return h_fin, xn_fin


# ------------------------------------------------------------------ routing --

@pytest.mark.parametrize("E,k", [(16, 4), (512, 4), (1024, 8), (5, 5), (64, 1)])
def test_route_topk_given_logits_exact(E, k):
    rng = np.random.default_rng(E * 10 + k)
    T = 7
    lg = rng.normal(size=(T, E)).astype(np.float32)
    lg[1] = 0.5                        # all tied
    lg[2, ::3] = 2.0                   # many tied maxima
    lg[3, 1:] = -np.arange(E - 1, dtype=np.float32)
    lg[4, 0] = np.float32(-0.0)
    lg[4, 1:] = 0.0                    # +0 / -0 tie
    logits = dev(lg)
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    fm.fmoe_route_topk(None, None, k, logits, ids, w, None, flags=fm.FMOE_LOGITS_GIVEN)
    ids_h, w_h = host(ids), host(w)
    for t in range(T):
        ri, rp, _ = oracle.topk_softmax(lg[t].astype(np.float64), k)
        assert ids_h[t].tolist() == ri.tolist(), (t, ids_h[t], ri)
        check(w_h[t], rp, rp, f"weights t={t}")
    assert fm.fmoe_read_status() == 0


def test_route_topk_nan_logits_set_status():
    E, k = 32, 4
    lg = np.linspace(1, 0, E, dtype=np.float32)[None].repeat(2, 0)
    lg[0, [0, 3]] = np.nan
    logits = dev(lg)
    ids = torch.empty((2, k), dtype=torch.int32, device="cuda")
    w = torch.empty((2, k), dtype=torch.float32, device="cuda")
    fm.fmoe_route_topk(None, None, k, logits, ids, w, None, flags=fm.FMOE_LOGITS_GIVEN)
    st = fm.fmoe_read_status(clear=True)
    assert st & fm.FMOE_STATUS_NAN_LOGIT
    for t in range(2):
        ri, rp, nan = oracle.topk_softmax(lg[t].astype(np.float64), k)
        assert host(ids)[t].tolist() == ri.tolist()
        check(host(w)[t], rp, rp, "weights")


@pytest.mark.parametrize("wl", [synth.TINY, synth.LAYER], ids=["tiny", "layer"])
def test_route_topk_router_product(wl):
    T = 3
    W = synth.router(wl, 2)
    x = synth.tokens(wl, T, stream=5)
    logits = torch.empty((T, wl.n_experts), device="cuda")
    ids = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), device="cuda")
    ws = fm.alloc_workspace(layer_desc(wl), T)
    fm.fmoe_route_topk(dev(x), dev(W), wl.top_k, logits, ids, w, ws)
    lg_h = host(logits)
    for t in range(T):
        lo, S = oracle.gemv_f32(W, x[t].astype(np.float64))
        check(lg_h[t], lo, S, "logits")
        ri, rp, _ = oracle.topk_softmax(lg_h[t].astype(np.float64), wl.top_k)
        assert host(ids)[t].tolist() == ri.tolist()
        check(host(w)[t], rp, rp, "weights")


# ------------------------------------------------------------ expert forward --

@pytest.mark.parametrize("wl", [synth.TINY, TINY2,
                                synth.Workload(n_experts=8), synth.Workload(n_experts=8, bits=2),
                                synth.Workload(hidden=2048, inter=512, n_experts=6, bits=4),
                                synth.Workload(hidden=128, inter=2048, n_experts=6, bits=4)],
                         ids=["tiny4", "tiny2", "full4", "full2", "h2048", "i2048"])
def test_expert_forward(wl):
    T = 3
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0)
    rng = np.random.default_rng(1)
    ids_h = np.stack([rng.choice(wl.n_experts, wl.top_k, replace=False) for _ in range(T)]).astype(np.int32)
    ids_h[2, 1] = ids_h[2, 0]  # a duplicate selection is legal
    x = synth.tokens(wl, T, stream=9)
    y = torch.empty((T, wl.top_k + 1, wl.hidden), device="cuda")
    gamma = torch.empty(T, device="cuda")
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_expert_forward(lw, dev(x), dev(ids_h), y, gamma, ws)
    y_h, g_h = host(y), host(gamma)
    for t in range(T):
        xd = x[t].astype(np.float64)
        for j, slot in enumerate(list(ids_h[t]) + [wl.n_experts]):
            ref = oracle.expert_ffn(lw_o.experts[int(slot)], wl.hidden, wl.inter, 64, xd)
            check(y_h[t, j], ref["y"], ref["S_y"], f"y t={t} j={j}")
        z, Sz = oracle.gemv_f32(lw_o.w_shared_gate[None], xd)
        gm = oracle.sigmoid(z[0])
        check(g_h[t], gm, gm + gm * (1 - gm) * Sz[0], "gamma")
    assert fm.fmoe_read_status() == 0


def test_expert_forward_bad_ids_set_status_and_zero_output():
    wl = synth.TINY
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0)
    ids_h = np.array([[3, -1, wl.n_experts, 7]], np.int32)
    x = synth.tokens(wl, 1, stream=11)
    y = torch.full((1, 5, wl.hidden), 7.0, device="cuda")
    gamma = torch.empty(1, device="cuda")
    ws = fm.alloc_workspace(lw.desc, 1)
    fm.fmoe_expert_forward(lw, dev(x), dev(ids_h), y, gamma, ws)
    st = fm.fmoe_read_status(clear=True)
    assert st & fm.FMOE_STATUS_BAD_EXPERT_ID
    y_h = host(y)
    assert np.all(y_h[0, 1] == 0) and np.all(y_h[0, 2] == 0)
    for j, slot in ((0, 3), (3, 7), (4, wl.n_experts)):
        ref = oracle.expert_ffn(lw_o.experts[slot], wl.hidden, wl.inter, 64, x[0].astype(np.float64))
        check(y_h[0, j], ref["y"], ref["S_y"], f"y j={j}")


# ------------------------------------------------------------------ combine --

@pytest.mark.parametrize("H,k,T", [(256, 4, 3), (4096, 4, 2), (4096, 8, 1), (64, 1, 5)])
def test_combine_residual_rmsnorm(H, k, T):
    rng = np.random.default_rng(H + k)
    y = rng.normal(size=(T, k + 1, H)).astype(np.float32) * 3
    p = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    gamma = rng.uniform(size=T).astype(np.float32)
    h = rng.normal(size=(T, H)).astype(np.float32)
    w = (1 + 0.1 * rng.normal(size=H)).astype(np.float32)
    h_out = torch.empty((T, H), device="cuda")
    xn_out = torch.empty((T, H), device="cuda")
    fm.fmoe_combine_residual_rmsnorm(dev(y), dev(p), dev(gamma), dev(h), dev(w), 1e-6, h_out, xn_out)
    for t in range(T):
        ho, xo, Sh, Sx = oracle.combine_rmsnorm(y[t], p[t], gamma[t], h[t], w, 1e-6)
        check(host(h_out)[t], ho, Sh, "h'")
        check(host(xn_out)[t], xo, Sx, "xn'")


def test_combine_in_place_residual():
    H, k, T = 256, 4, 2
    rng = np.random.default_rng(3)
    y = rng.normal(size=(T, k + 1, H)).astype(np.float32)
    p = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    gamma = rng.uniform(size=T).astype(np.float32)
    h = rng.normal(size=(T, H)).astype(np.float32)
    w = np.ones(H, np.float32)
    hd = dev(h)
    xn_out = torch.empty((T, H), device="cuda")
    fm.fmoe_combine_residual_rmsnorm(dev(y), dev(p), dev(gamma), hd, dev(w), 1e-6, hd, xn_out)
    for t in range(T):
        ho, xo, Sh, Sx = oracle.combine_rmsnorm(y[t], p[t], gamma[t], h[t], w, 1e-6)
        check(host(hd)[t], ho, Sh, "h' in place")
        check(host(xn_out)[t], xo, Sx, "xn'")


# -------------------------------------------------------------- layer forward --

@pytest.fixture(params=[True, False], ids=["fused", "per-step"])
def path(request):
    prev = fm.fmoe_set_fused(request.param)
    yield request.param
    fm.fmoe_set_fused(prev)


@pytest.mark.parametrize("wl,T", [(synth.TINY, 1), (synth.TINY, 3), (TINY2, 1), (TINY2, 2), (SMALL, 1), (SMALL2, 1),
                                  (SMALL, 2)],
                         ids=["tiny-T1", "tiny-T3", "tiny2-T1", "tiny2-T2", "small-T1", "small2-T1", "small-T2"])
def test_layer_forward_tiny(wl, T, path):
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0)
    x = synth.tokens(wl, T, stream=21)
    h = dev(x)
    xn = dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward(lw, h, xn, ws)
    for t in range(T):
        check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], host(h)[t], host(xn)[t], f"t={t}")
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("wl,T", [(synth.Workload(hidden=1024, inter=512, n_experts=1024, top_k=8), 1),
                                  (synth.Workload(hidden=1024, inter=512, n_experts=1024, top_k=8), 6),
                                  (synth.Workload(hidden=256, inter=256, n_experts=64, top_k=1), 1),
                                  (synth.Workload(hidden=256, inter=256, n_experts=64, top_k=1), 3),
                                  (synth.Workload(hidden=256, inter=256, n_experts=4, top_k=4), 1),
                                  (synth.Workload(hidden=256, inter=256, n_experts=4, top_k=4), 2)],
                         ids=["E1024-k8-T1", "E1024-k8-T6", "k1-T1", "k1-T3", "k=E-T1", "k=E-T2"])
def test_layer_forward_routing_extremes(wl, T, path):
    """The largest routing the library takes (1024 experts, top-8; the
    persistent kernel's router rows do not cover it, so the one-kernel-per-
    step path runs), top-1, and every expert selected (k = E): every output
    of every token against the oracle."""
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0, slots=[wl.n_experts])
    x = synth.tokens(wl, T, stream=71)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward(lw, h, xn, ws)
    pmap(lambda t: check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], host(h)[t], host(xn)[t], f"t={t}"),
         range(T))
    assert fm.fmoe_read_status() == 0


@pytest.fixture(scope="module")
def full_layer():
    wl = synth.LAYER
    return wl, device_layer(wl, 0), oracle_layer(wl, 0, slots=[wl.n_experts])


def test_layer_forward_full_size(full_layer, path):
    """One 4-bit layer at hidden 4096 / 512 experts, batch 1, every output checked."""
    wl, lw, lw_o = full_layer
    x = synth.tokens(wl, 1, stream=31)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, 1)
    fm.fmoe_layer_forward(lw, h, xn, ws)
    check_layer_token(wl, lw_o, ws, lw.desc, 1, 0, x[0], x[0], host(h)[0], host(xn)[0], "full")
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("wl", [synth.Workload(n_experts=32, bits=2)], ids=["int2-32"])
def test_layer_forward_full_size_int2(wl, path):
    """hidden 4096 / inter 1024 with 2-bit routed experts (4-bit shared), batch 1."""
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0, slots=[wl.n_experts])
    for stream in (33, 34):
        x = synth.tokens(wl, 1, stream=stream)
        h, xn = dev(x), dev(x)
        ws = fm.alloc_workspace(lw.desc, 1)
        fm.fmoe_layer_forward(lw, h, xn, ws)
        check_layer_token(wl, lw_o, ws, lw.desc, 1, 0, x[0], x[0], host(h)[0], host(xn)[0], f"int2 {stream}")
    assert fm.fmoe_read_status() == 0


def test_fused_and_per_step_paths_agree(full_layer):
    """The persistent kernel and the one-kernel-per-step path route alike and
    agree to well inside the oracle tolerance.  They are not bit-identical:
    the persistent kernel stages the SwiGLU outputs as 24-bit block floating
    point per column block of 8 units, the per-step path per 64-group, and it
    sums the expert outputs in another order."""
    wl, lw, _ = full_layer
    x = synth.tokens(wl, 1, stream=35)
    outs = {}
    for fused in (True, False):
        prev = fm.fmoe_set_fused(fused)
        h, xn = dev(x), dev(x)
        ws = fm.alloc_workspace(lw.desc, 1)
        fm.fmoe_layer_forward(lw, h, xn, ws)
        outs[fused] = (host(h)[0], host(xn)[0], host(fm.workspace_view(ws, lw.desc, 1, fm.WS_A))[0],
                       host(fm.workspace_view(ws, lw.desc, 1, fm.WS_IDS))[0])
        fm.fmoe_set_fused(prev)
    assert outs[True][3].tolist() == outs[False][3].tolist()
    for i in range(3):
        a, b = outs[True][i], outs[False][i]
        assert np.linalg.norm(a - b) / np.linalg.norm(b) < 2e-4, i


def test_layer_forward_is_deterministic_and_graph_capturable(full_layer):
    wl, lw, _ = full_layer
    x = synth.tokens(wl, 1, stream=32)
    ws = fm.alloc_workspace(lw.desc, 1)
    outs = []
    for _ in range(2):
        h, xn = dev(x), dev(x)
        fm.fmoe_layer_forward(lw, h, xn, ws)
        outs.append((host(h), host(xn)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    h, xn = dev(x), dev(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fm.fmoe_layer_forward(lw, h, xn, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    h.copy_(dev(x))
    xn.copy_(dev(x))
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(host(h), outs[0][0]) and np.array_equal(host(xn), outs[0][1])


def test_layer_forward_batched_zipf_routing(full_layer, tc_path):
    """64 tokens through one layer on Zipf(1)-popularity Gumbel-top-k routing
    logits; every token checked against the oracle (hot experts and the
    shared expert on the tensor cores, or all on the integer-dot path)."""
    wl, lw, lw_o = full_layer
    T = 64
    lg, _ = synth.zipf_gumbel_logits(wl, 0, T)
    x = synth.tokens(wl, T, stream=41)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward_logits(lw, dev(lg), h, xn, ws)
    ids_d = host(fm.workspace_view(ws, lw.desc, T, fm.WS_IDS))
    counts = np.bincount(ids_d.ravel(), minlength=wl.n_experts)
    assert counts.max() >= 16  # Zipf routing gives hot experts
    h_d, xn_d = host(h), host(xn)

    def one(t):
        ri, _, _ = oracle.topk_softmax(lg[t].astype(np.float64), wl.top_k)
        assert ri.tolist() == ids_d[t].tolist()
        check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], h_d[t], xn_d[t], f"t={t}", logits_given=True)

    pmap(one, range(T))


@pytest.fixture(params=[True, False], ids=["tensor-cores", "integer-dot"])
def tc_path(request):
    prev = fm.fmoe_set_tensor_cores(request.param)
    yield request.param
    fm.fmoe_set_tensor_cores(prev)


@pytest.mark.parametrize("wl", [SMALL, SMALL2], ids=["small4", "small2"])
def test_grouped_experts_many_tokens_per_expert(wl, tc_path):
    """40 tokens all routed to the same four experts (given logits): every
    group holds 40 slots -- a dense product on the tensor cores, or work
    items of up to 16 tokens on the integer-dot path.  Tokens from each
    item, and the last one, are checked against the oracle."""
    T = 40
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0)
    lg = np.zeros((T, wl.n_experts), np.float32)
    lg[:, [3, 7, 11, 15]] = [4.0, 3.0, 2.0, 1.0]
    x = synth.tokens(wl, T, stream=43)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward_logits(lw, dev(lg), h, xn, ws)
    for t in (0, 15, 16, 31, 32, 39):
        check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], host(h)[t], host(xn)[t], f"t={t}",
                          logits_given=True)
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("wl", [synth.Workload(n_experts=32, bits=2)], ids=["int2-32"])
def test_batched_full_size_int2_every_item_size(wl, tc_path):
    """hidden 4096 / inter 1024, 2-bit routed experts, 24 tokens on given
    logits chosen so that every kind of work item occurs: experts with 2
    tokens and with 3 tokens (the bulk-copied small-item GEMV), 4-5 tokens
    and 6 and 24 tokens (tensor cores from 5 tokens on), and the 4-bit
    shared expert with all 24; sampled tokens checked against the oracle."""
    T = 24
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0, slots=[wl.n_experts])
    lg = np.zeros((T, wl.n_experts), np.float32)
    for t in range(T):
        picks = [0, 1 if t < 6 else 2 + t % 4, 10 + t % 8, 20 + t % 12]
        lg[t, picks] = [4.0, 3.0, 2.0, 1.0]
    counts = np.bincount(np.argsort(-lg, axis=1)[:, :4].ravel(), minlength=wl.n_experts)
    assert {2, 3, 6, 24} <= set(counts.tolist()) and (counts[2:6] >= 4).all()
    x = synth.tokens(wl, T, stream=47)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward_logits(lw, dev(lg), h, xn, ws)
    for t in (0, 5, 6, 13, 23):
        check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], host(h)[t], host(xn)[t], f"t={t}",
                          logits_given=True)
    assert fm.fmoe_read_status() == 0


def _run(lws, x, stack):
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lws[0].desc, len(x))
    if stack:
        fm.fmoe_stack_forward(lws, h, xn, ws)
    else:
        fm.fmoe_layer_forward(lws[0], h, xn, ws)
    return host(h), host(xn), ws


@pytest.mark.parametrize("wl", [synth.TINY, SMALL], ids=["tiny4", "small4"])
def test_few_tokens_through_persistent_kernel(wl):
    """Up to fmoe_fused_max_tokens tokens run through the persistent kernel,
    two per launch (4-bit layers): every token of a layer call, and every
    layer of every token of a traced stack call, against the oracle; a
    token's bits do not depend on its partner in the pair; an odd last
    token gets the bits of a T = 1 call; one token more than the maximum
    takes the grouped path and agrees within the tolerance."""
    if not fm.fmoe_fused_supported(device_layer(wl).desc):
        pytest.skip("persistent kernel does not fit this shape here")
    n_layers = 3
    lws = [device_layer(wl, l) for l in range(n_layers)]
    los = [oracle_layer(wl, l) for l in range(n_layers)]
    for l, lo in enumerate(los):
        lo.layer = l
    Tl, Ts = fm.fmoe_fused_max_tokens(False), fm.fmoe_fused_max_tokens(True)
    x = synth.tokens(wl, Ts + 2, stream=61)
    # layer calls of Tl tokens (pairs), chained over the layers, each against the oracle
    h, xn = dev(x[:Tl]), dev(x[:Tl])
    ws = fm.alloc_workspace(lws[0].desc, Tl)
    for l in range(n_layers):
        h_in, xn_in = host(h), host(xn)
        fm.fmoe_layer_forward(lws[l], h, xn, ws)
        for t in range(Tl):
            check_layer_token(wl, los[l], ws, lws[l].desc, Tl, t, h_in[t], xn_in[t], host(h)[t], host(xn)[t],
                              f"layer {l} t={t}")
    # the stack over Ts tokens, every layer of every token checked on its trace
    traced_stack_check(wl, lws, los, x[:Ts], "few tokens")
    for stack in (False, True):
        T = Ts if stack else Tl
        got_h, got_xn, _ = _run(lws, x[:T], stack)
        # partner independence: token 0 paired with token T instead of token 1
        xp = x[:T].copy()
        xp[1] = x[T]
        ph, pxn, _ = _run(lws, xp, stack)
        assert np.array_equal(ph[0], got_h[0]) and np.array_equal(pxn[0], got_xn[0]), stack
        assert not np.array_equal(pxn[1], got_xn[1])
        one = [_run(lws, x[t:t + 1], stack) for t in range(T + 1)]
        # an odd last token runs alone: the bits of a T = 1 call
        oh, oxn, _ = _run(lws, x[:3], stack)
        assert np.array_equal(oh[2], one[2][0][0]) and np.array_equal(oxn[2], one[2][1][0]), stack
        for t in range(T):
            rel = np.linalg.norm(got_xn[t] - one[t][1][0]) / np.linalg.norm(one[t][1][0])
            assert rel <= 2e-3, (stack, t, rel)
        # one token more: the grouped path
        gh, gxn, _ = _run(lws, x[:T + 1], stack)
        for t in range(T + 1):
            rel = np.linalg.norm(gxn[t] - one[t][1][0]) / np.linalg.norm(one[t][1][0])
            assert rel <= 2e-3, (stack, t, rel)
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("wl", [SMALL, SMALL2], ids=["small4", "small2"])
def test_stack_trace_beyond_persistent_tokens(wl):
    """A traced stack of more tokens than the persistent kernel takes (the
    grouped path, layer by layer, the trace copied from the workspace):
    every layer of every token against the oracle, and the traced stack
    gives the bits of the untraced one."""
    L = 3
    lws = [device_layer(wl, l) for l in range(L)]
    los = [oracle_layer(wl, l) for l in range(L)]
    for l, lo in enumerate(los):
        lo.layer = l
    T = fm.fmoe_fused_max_tokens(True) + 2
    x = synth.tokens(wl, T, stream=67)
    h_t, xn_t = traced_stack_check(wl, lws, los, x, "grouped")
    h, xn = dev(x), dev(x)
    fm.fmoe_stack_forward(lws, h, xn, fm.alloc_workspace(lws[0].desc, T))
    assert np.array_equal(host(h), h_t) and np.array_equal(host(xn), xn_t)
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("T", [1, 3, 6])
def test_host_state_entry_point_matches_device_entry_point(T):
    """fmoe_layer_forward_host (pinned host h/xn in, h'/xn' out, one copy
    each way) gives the bits of fmoe_layer_forward on device tensors."""
    wl = SMALL
    lw = device_layer(wl)
    x = synth.tokens(wl, T, stream=63)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward(lw, h, xn, ws)
    hx_in = torch.from_numpy(np.stack([x, x])).pin_memory()
    hx_out = torch.zeros_like(hx_in).pin_memory()
    d_hx = torch.empty(hx_in.shape, dtype=torch.float32, device="cuda")
    ws2 = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward_host(lw, hx_in, hx_out, d_hx, ws2)
    torch.cuda.synchronize()
    assert np.array_equal(hx_out[0].numpy(), host(h)) and np.array_equal(hx_out[1].numpy(), host(xn))
    assert fm.fmoe_read_status() == 0


@pytest.mark.parametrize("T", [1, 2])
def test_host_state_stack_matches_device_stack(T):
    """fmoe_stack_forward_host (pinned host h/xn in, three layers, h'/xn'
    out) gives the bits of fmoe_stack_forward on device tensors."""
    wl = SMALL
    lws = [device_layer(wl, l) for l in range(3)]
    x = synth.tokens(wl, T, stream=64)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lws[0].desc, T)
    fm.fmoe_stack_forward(lws, h, xn, ws)
    hx = torch.from_numpy(np.stack([x, x])).pin_memory()
    d_hx = torch.empty(hx.shape, dtype=torch.float32, device="cuda")
    ws2 = fm.alloc_workspace(lws[0].desc, T)
    fm.fmoe_stack_forward_host(lws, hx, hx, d_hx, ws2)  # in place on the host buffer
    torch.cuda.synchronize()
    assert np.array_equal(hx[0].numpy(), host(h)) and np.array_equal(hx[1].numpy(), host(xn))
    assert fm.fmoe_read_status() == 0


def test_tensor_core_and_integer_paths_differ_only_by_rounding():
    """The two implementations of the grouped products both run (their
    results are not bit-identical) and agree well inside the tolerance."""
    wl = SMALL
    T = 40
    lw = device_layer(wl)
    lg = np.zeros((T, wl.n_experts), np.float32)
    lg[:, [2, 5, 9, 13]] = [4.0, 3.0, 2.0, 1.0]
    x = synth.tokens(wl, T, stream=44)
    outs = {}
    for tc in (True, False):
        prev = fm.fmoe_set_tensor_cores(tc)
        h, xn = dev(x), dev(x)
        ws = fm.alloc_workspace(lw.desc, T)
        fm.fmoe_layer_forward_logits(lw, dev(lg), h, xn, ws)
        outs[tc] = (host(fm.workspace_view(ws, lw.desc, T, fm.WS_A)), host(fm.workspace_view(ws, lw.desc, T, fm.WS_Y)))
        fm.fmoe_set_tensor_cores(prev)
    for i in range(2):
        a, b = outs[True][i], outs[False][i]
        assert not np.array_equal(a, b)
        assert np.linalg.norm(a - b) / np.linalg.norm(b) < 1e-3


# ------------------------------------------------------------------- chains --

@pytest.mark.parametrize("wl", [synth.TINY, TINY2, SMALL, SMALL2], ids=["tiny4", "tiny2", "small4", "small2"])
def test_stack_chain_teacher_forced_and_free_running(wl, path):
    """A 4-layer stack decoding 3 tokens, each next token starting from the
    previous token's final xn'.  Layer by layer (fmoe_layer_forward) and as
    one traced stack call per token: every layer checked teacher-forced on
    the device's inputs; the stack gives the bits of the layer calls; the
    decode agrees with the free-running fp64 chain in relative L2."""
    L, steps = 4, 3
    lws = [device_layer(wl, l) for l in range(L)]
    los = [oracle_layer(wl, l) for l in range(L)]
    for l, lo in enumerate(los):
        lo.layer = l
    x0 = synth.tokens(wl, 1, stream=51)[0]
    ws = fm.alloc_workspace(lws[0].desc, 1)
    # layer by layer
    tok = x0.copy()
    h, xn = dev(tok[None]), dev(tok[None])
    free_h = tok.astype(np.float64)
    free_xn = tok.astype(np.float64)
    first = None
    for s in range(steps):
        for l in range(L):
            h_in, xn_in = host(h)[0], host(xn)[0]
            fm.fmoe_layer_forward(lws[l], h, xn, ws)
            if s == 0 and l == 0:
                first = (host(h)[0], host(xn)[0])
            check_layer_token(wl, los[l], ws, lws[l].desc, 1, 0, h_in, xn_in, host(h)[0], host(xn)[0],
                              f"step {s} layer {l}")
            ref = oracle.layer_token(wl, los[l], free_h, free_xn, expert_fn=lambda e, l=l: synth.expert(wl, l, e))
            free_h, free_xn = ref["h"], ref["xn"]
        h.copy_(xn)
        free_h = free_xn.copy()
    final_layered = host(xn)[0]
    rel = np.linalg.norm(final_layered - free_xn) / np.linalg.norm(free_xn)
    assert rel <= 2e-3, rel
    # the stack entry point, traced, one call per token: the same bits
    tok = x0.copy()
    for s in range(steps):
        if s == 0:
            tr = fm.alloc_trace(lws[0].desc, 1, 1)
            h1, xn1 = dev(tok[None]), dev(tok[None])
            fm.fmoe_stack_forward(lws[:1], h1, xn1, ws, trace=tr)
            assert np.array_equal(host(h1)[0], first[0]) and np.array_equal(host(xn1)[0], first[1])
        _, xn_s = traced_stack_check(wl, lws, los, tok[None], f"step {s}")
        tok = xn_s[0].copy()
    assert np.array_equal(tok, final_layered)
    assert fm.fmoe_read_status() == 0


# ---------------------------------------------------------- outlier inputs --

def outlier_tokens(wl, T, stream):
    """Tokens whose groups of 64 inputs span a wide range: every group has
    one channel scaled by 300 (a residual-stream outlier), and every fourth
    group is scaled by 1e-4 as a whole.  The device stages each group with
    one power-of-two step; these inputs put the step far from most of the
    group's values."""
    x = synth.tokens(wl, T, stream=stream).astype(np.float32)
    G = 64
    for g in range(wl.hidden // G):
        x[:, g * G + (7 * g) % G] *= 300.0
        if g % 4 == 3:
            x[:, g * G:(g + 1) * G] *= 1e-4
    return x


@pytest.mark.parametrize("wl", [synth.TINY, synth.LAYER], ids=["tiny", "full"])
def test_layer_forward_outlier_activations(wl, path):
    """Activation outliers at batch 1 through the persistent kernel and the
    one-kernel-per-step path: every output of the layer within the oracle's
    tolerance, element by element."""
    lw = device_layer(wl)
    lw_o = oracle_layer(wl, 0, slots=None if wl.n_experts <= 16 else [wl.n_experts])
    x = outlier_tokens(wl, 2, stream=71)
    for t in range(2):
        h, xn = dev(x[t:t + 1]), dev(x[t:t + 1])
        ws = fm.alloc_workspace(lw.desc, 1)
        fm.fmoe_layer_forward(lw, h, xn, ws)
        check_layer_token(wl, lw_o, ws, lw.desc, 1, 0, x[t], x[t], host(h)[0], host(xn)[0], f"outliers t={t}")
    assert fm.fmoe_read_status() == 0


def test_batched_outlier_activations(full_layer, tc_path):
    """The same outliers through the grouped T > 1 path (integer-dot GEMV
    and tensor cores) with routing on the router product."""
    wl, lw, lw_o = full_layer
    T = 12
    x = outlier_tokens(wl, T, stream=73)
    h, xn = dev(x), dev(x)
    ws = fm.alloc_workspace(lw.desc, T)
    fm.fmoe_layer_forward(lw, h, xn, ws)
    h_d, xn_d = host(h), host(xn)
    pmap(lambda t: check_layer_token(wl, lw_o, ws, lw.desc, T, t, x[t], x[t], h_d[t], xn_d[t], f"t={t}"), range(T))
    assert fm.fmoe_read_status() == 0
