"""Host-memory expert tier with a device cache (fmoe_cache_*): results equal
the resident-weights layer bit for bit, and the hit / miss accounting follows
least-recently-used replacement."""
import numpy as np
import pytest
import torch

import synth
from synth.device import upload_layer

pytestmark = pytest.mark.gpu

fm = pytest.importorskip("quantized_expert_gemv_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


SMALL = synth.Workload(hidden=256, inter=256, n_experts=16)


def _layers(wl, n):
    lws = [upload_layer(wl, l) for l in range(n)]
    host = [lw.experts.cpu().pin_memory() for lw in lws]
    return lws, host


@pytest.mark.parametrize("T", [1, 3, 6])
def test_cached_layers_equal_resident_layers(T):
    """Three layers, six slots (fewer than the experts the steps touch, so
    records are evicted and copied back), five steps: every step's h', xn'
    equal the one-kernel-per-step path on resident weights bit for bit."""
    wl = SMALL
    lws, host = _layers(wl, 3)
    cache = fm.ExpertCache(lws[0].desc, host, n_slots=max(6, T * wl.top_k), max_tokens=T)
    x = synth.tokens(wl, T, stream=71)
    h_c, xn_c = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
    h_r, xn_r = h_c.clone(), xn_c.clone()
    ws_c, ws_r = fm.alloc_workspace(lws[0].desc, T), fm.alloc_workspace(lws[0].desc, T)
    prev = fm.fmoe_set_fused(False)
    try:
        for step in range(5):
            for l in range(3):
                cache.forward(l, lws[l], h_c, xn_c, ws_c)
                fm.fmoe_layer_forward(lws[l], h_r, xn_r, ws_r)
                torch.cuda.synchronize()
                assert torch.equal(h_c, h_r) and torch.equal(xn_c, xn_r), (step, l)
            h_c.copy_(xn_c)
            h_r.copy_(xn_r)
    finally:
        fm.fmoe_set_fused(prev)
    hits, misses, nbytes = cache.stats()
    assert misses >= 1 and nbytes == misses * lws[0].desc.record_bytes()
    assert fm.fmoe_read_status() == 0
    cache.close()


def _lru_reference(steps, n_slots):
    """Least recently used replacement over (layer, id) keys in numbered
    slots: an empty slot first (lowest number), else the lowest-numbered of
    the least recently used slots not touched by the current step."""
    key = [None] * n_slots
    stamp = [0] * n_slots
    hits = misses = clock = 0
    for layer, ids in steps:
        clock += 1
        for e in ids:
            k = (layer, int(e))
            if k in key:
                s = key.index(k)
                if stamp[s] < clock:
                    hits += 1
                stamp[s] = clock
                continue
            free = [s for s in range(n_slots) if key[s] is None]
            if free:
                s = free[0]
            else:
                cand = [s for s in range(n_slots) if stamp[s] < clock]
                s = min(cand, key=lambda i: (stamp[i], i))
            key[s], stamp[s] = k, clock
            misses += 1
    return hits, misses


def test_cache_accounting_follows_lru():
    """Given routing (logits) with a scripted id sequence over two layers:
    the cache's hits and misses match a least-recently-used reference."""
    wl = SMALL
    lws, host = _layers(wl, 2)
    n_slots, T = 9, 2
    cache = fm.ExpertCache(lws[0].desc, host, n_slots=n_slots, max_tokens=T)
    r = np.random.default_rng(5)
    steps, logit_steps = [], []
    for s in range(24):
        layer = s % 2
        lg = np.zeros((T, wl.n_experts), np.float32)
        chosen = []
        for t in range(T):
            ids = r.choice(6 if s % 3 else wl.n_experts, size=wl.top_k, replace=False)  # skewed: mostly experts 0-5
            lg[t, ids] = [4.0, 3.0, 2.0, 1.0]
            chosen.extend(ids.tolist())
        steps.append((layer, chosen))
        logit_steps.append(lg)
    x = synth.tokens(wl, T, stream=72)
    h, xn = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
    ws = fm.alloc_workspace(lws[0].desc, T)
    for (layer, _), lg in zip(steps, logit_steps):
        cache.forward(layer, lws[layer], h, xn, ws, logits=torch.from_numpy(lg).cuda())
    torch.cuda.synchronize()
    hits, misses, _ = cache.stats()
    want = _lru_reference(steps, n_slots)
    assert (hits, misses) == want
    assert fm.fmoe_read_status() == 0
    cache.close()


def test_cache_too_small_for_one_step_is_an_error():
    wl = SMALL
    lws, host = _layers(wl, 1)
    cache = fm.ExpertCache(lws[0].desc, host, n_slots=3, max_tokens=1)
    x = synth.tokens(wl, 1, stream=73)
    h, xn = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
    ws = fm.alloc_workspace(lws[0].desc, 1)
    with pytest.raises(fm.FmoeError):
        cache.forward(0, lws[0], h, xn, ws)
    cache.close()


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("fused", [True, False], ids=["fused-enabled", "fused-disabled"])
def test_cached_steps_match_oracle(T, fused):
    """Cached layer steps against the fp64 oracle, element by element: the
    router logits, the top-k on the device's logits, the gate weights and
    gamma, every selected expert's SwiGLU outputs a and down outputs y, h'
    and xn'.  Two steps per layer: the first copies its records in from host
    memory, the second finds them in the cache.  The host tier runs the same
    way with the persistent kernel enabled or not (it learns the routing on
    the host before the expert products, so it always takes the
    one-kernel-per-step products)."""
    import oracle
    from tests.parity import check
    wl = SMALL
    lws, host = _layers(wl, 2)
    cache = fm.ExpertCache(lws[0].desc, host, n_slots=max(6, T * wl.top_k), max_tokens=T)
    x = synth.tokens(wl, T, stream=74)
    h, xn = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
    ws = fm.alloc_workspace(lws[0].desc, T)
    prev = fm.fmoe_set_fused(fused)
    try:
        for step in range(2):
            for l in range(2):
                h_in, xn_in = h.cpu().numpy().astype(np.float64), xn.cpu().numpy().astype(np.float64)
                cache.forward(l, lws[l], h, xn, ws)
                torch.cuda.synchronize()
                view = lambda which: fm.workspace_view(ws, lws[l].desc, T, which).cpu().numpy()
                lg, ids, p, gm = view(fm.WS_LOGITS), view(fm.WS_IDS), view(fm.WS_WEIGHTS), view(fm.WS_GAMMA)
                a, y = view(fm.WS_A), view(fm.WS_Y)
                lo = oracle.LayerWeights(synth.router(wl, l), synth.shared_gate(wl, l), synth.norm_weight(wl, l),
                                         {e: synth.expert(wl, l, e) for e in range(wl.n_experts + 1)})
                for t in range(T):
                    label = f"step {step} layer {l} token {t}"
                    lg_o, S_l = oracle.gemv_f32(lo.w_router, xn_in[t])
                    check(lg[t], lg_o, S_l, f"{label} logits")
                    ref = oracle.layer_token(wl, lo, h_in[t], xn_in[t], logits_in=lg[t])
                    assert ref["ids"].tolist() == ids[t].tolist(), label
                    check(p[t], ref["p"], ref["p"], f"{label} gate weights")
                    check(gm[t], ref["gamma"], ref["gamma"] + ref["S_gamma"], f"{label} gamma", rel_l2=False)
                    for j, slot in enumerate(list(ids[t]) + [wl.n_experts]):
                        e = oracle.expert_ffn(lo.experts[int(slot)], wl.hidden, wl.inter, 64, xn_in[t])
                        check(a[t, j], e["a"], e["S_a"], f"{label} a[{j}]")
                    check(y[t], ref["y"], ref["S_y"], f"{label} y")
                    check(h.cpu().numpy()[t], ref["h"], ref["S_h"], f"{label} h'")
                    check(xn.cpu().numpy()[t], ref["xn"], ref["S_xn"], f"{label} xn'")
            h.copy_(xn)
    finally:
        fm.fmoe_set_fused(prev)
    hits, misses, _ = cache.stats()
    assert hits >= 1 and misses >= 1
    assert fm.fmoe_read_status() == 0
    cache.close()
