"""Pins of the CPU oracle against facts other than its own formulas.

Each test reduces the oracle to a case whose answer is fixed independently:
closed forms, integer arithmetic, algebraic identities stated by the pages
("What is Flash-MoE?", section "2. FMA-optimised dequantisation kernels":
(code * scale + bias) * x = code * (scale * x) + bias * x), invariants
(relabelling experts), the quantiser's round trip, and the byte counts the
pages print (tests/golden/pages_figures.txt).  A dropped term, a wrong sign,
a transposed operand or a wrong group index in the oracle fails one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.txt")

BF16_ONE = 0x3F80


def bf16_pow2(k: int) -> int:
    """bf16 bit pattern of 2**k (exact)."""
    return (127 + k) << 7


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- GEMV ----

def test_qgemv_unit_scale_zero_bias_sums_codes():
    r = rng(1)
    q = r.integers(0, 16, size=(37, 192), dtype=np.uint8)
    s = np.full((37, 3), BF16_ONE, np.uint16)
    b = np.zeros((37, 3), np.uint16)
    y, S = oracle.qgemv(q, s, b, 64, np.ones(192))
    assert np.array_equal(y, q.astype(np.int64).sum(1).astype(np.float64))
    assert np.array_equal(S, y)  # all terms non-negative


def test_qgemv_power_of_two_scale_integer_x_is_exact():
    r = rng(2)
    rows, cols, G = 11, 256, 64
    q = r.integers(0, 16, size=(rows, cols), dtype=np.uint8)
    ks = r.integers(-12, -2, size=(rows, cols // G))
    s = np.vectorize(bf16_pow2)(ks).astype(np.uint16)
    b = np.zeros_like(s)
    x = r.integers(-50, 50, size=cols)
    y, _ = oracle.qgemv(q, s, b, G, x.astype(np.float64))
    # exact rational answer with integer arithmetic: sum_g 2^k_g * sum_j q x
    for i in range(rows):
        tot = 0.0
        for g in range(cols // G):
            part = int((q[i, g * G:(g + 1) * G].astype(np.int64) * x[g * G:(g + 1) * G]).sum())
            tot += math.ldexp(part, int(ks[i, g]))
        assert y[i] == tot


def test_qgemv_zero_codes_gives_bias_times_group_sums():
    r = rng(3)
    rows, cols, G = 5, 128, 64
    q = np.zeros((rows, cols), np.uint8)
    s = synth.f32_to_bf16(r.uniform(0.005, 0.02, size=(rows, 2)).astype(np.float32))
    b = synth.f32_to_bf16(r.normal(size=(rows, 2)).astype(np.float32))
    x = np.ones(cols)
    x[:G] = 0.5  # group sums 32 and 64
    y, _ = oracle.qgemv(q, s, b, G, x)
    bv = synth.bf16_to_f32(b).astype(np.float64)
    assert np.allclose(y, bv[:, 0] * 32 + bv[:, 1] * 64, rtol=0, atol=1e-12)


def test_qgemv_one_hot_reads_single_weight():
    r = rng(4)
    rows, cols, G = 6, 192, 64
    q = r.integers(0, 16, size=(rows, cols), dtype=np.uint8)
    s = synth.f32_to_bf16(r.uniform(0.005, 0.02, size=(rows, 3)).astype(np.float32))
    b = synth.f32_to_bf16(r.normal(0, 0.1, size=(rows, 3)).astype(np.float32))
    sv, bv = synth.bf16_to_f32(s).astype(np.float64), synth.bf16_to_f32(b).astype(np.float64)
    for j in (0, 63, 64, 130, 191):
        x = np.zeros(cols)
        x[j] = 1.0
        y, _ = oracle.qgemv(q, s, b, G, x)
        # weight (row i, column j) = code * scale of group j // 64 + bias of that group
        expect = q[:, j] * sv[:, j // G] + bv[:, j // G]
        assert np.array_equal(y, expect)


def test_qgemv_fma_identity_of_the_pages():
    """(q s + b) x summed == sum_g s_g (sum_j q_j x_j) + b_g (sum_j x_j)."""
    wl = synth.TINY
    ex = synth.expert(wl, 0, 3)
    (qg, sg, bg), _, _ = ex.matrices(wl)
    x = synth.tokens(wl, 1)[0].astype(np.float64)
    y, S = oracle.qgemv(qg, sg, bg, 64, x)
    sv, bv = synth.bf16_to_f32(sg).astype(np.float64), synth.bf16_to_f32(bg).astype(np.float64)
    ng = qg.shape[1] // 64
    qx = (qg.astype(np.float64) * x).reshape(qg.shape[0], ng, 64).sum(2)
    X = x.reshape(ng, 64).sum(1)
    fact = (sv * qx + bv * X).sum(1)
    assert np.allclose(y, fact, rtol=1e-12, atol=1e-12 * S.max())


def test_qgemv_linear_in_x_and_row_permutation():
    r = rng(5)
    q = r.integers(0, 4, size=(9, 128), dtype=np.uint8)
    s = synth.f32_to_bf16(r.uniform(0.02, 0.08, size=(9, 2)).astype(np.float32))
    b = synth.f32_to_bf16(r.normal(size=(9, 2)).astype(np.float32))
    x1, x2 = r.normal(size=128), r.normal(size=128)
    y1, S1 = oracle.qgemv(q, s, b, 64, x1)
    y2, S2 = oracle.qgemv(q, s, b, 64, x2)
    y12, _ = oracle.qgemv(q, s, b, 64, x1 + x2)
    assert np.allclose(y12, y1 + y2, rtol=0, atol=1e-12 * (S1 + S2).max())
    perm = r.permutation(9)
    yp, _ = oracle.qgemv(q[perm], s[perm], b[perm], 64, x1)
    assert np.array_equal(yp, y1[perm])


def test_qgemv_brute_force_dense_on_tiny():
    """Dequantise with a lookup table over every (code, group) pair, then a
    dense matmul -- a different route to the same numbers."""
    r = rng(6)
    rows, cols, G = 8, 128, 64
    q = r.integers(0, 16, size=(rows, cols), dtype=np.uint8)
    s = synth.f32_to_bf16(r.uniform(0.005, 0.02, size=(rows, 2)).astype(np.float32))
    b = synth.f32_to_bf16(r.normal(0, 0.01, size=(rows, 2)).astype(np.float32))
    table = (np.arange(16)[None, None, :] * synth.bf16_to_f32(s).astype(np.float64)[:, :, None]
             + synth.bf16_to_f32(b).astype(np.float64)[:, :, None])  # [rows][groups][code]
    W = np.empty((rows, cols))
    for i in range(rows):
        for j in range(cols):
            W[i, j] = table[i, j // G, q[i, j]]
    x = r.normal(size=cols)
    y, S = oracle.qgemv(q, s, b, G, x)
    assert np.allclose(y, W @ x, rtol=0, atol=1e-13 * S.max())
    assert np.allclose(S, np.abs(W * x).sum(1), rtol=1e-14)


def test_gemv_f32_identity_and_ones():
    x = rng(7).normal(size=32)
    y, _ = oracle.gemv_f32(np.eye(32, dtype=np.float32), x)
    assert np.array_equal(y, x)
    y, S = oracle.gemv_f32(np.ones((3, 32), np.float32), x)
    assert np.allclose(y, x.sum(), rtol=1e-15) and np.allclose(S, np.abs(x).sum())


# -------------------------------------------------------------- routing ----

def test_topk_strictly_decreasing_selects_first_four():
    ids, p, nan = oracle.topk_softmax(-np.arange(512.0), 4)
    assert ids.tolist() == [0, 1, 2, 3] and not nan
    # softmax of (0, -1, -2, -3), closed form
    z = sum(math.exp(-t) for t in range(4))
    assert np.allclose(p, [math.exp(-t) / z for t in range(4)], rtol=1e-15)


def test_topk_all_equal_breaks_ties_to_lowest_index():
    ids, p, _ = oracle.topk_softmax(np.full(512, 0.3), 4)
    assert ids.tolist() == [0, 1, 2, 3]
    assert np.array_equal(p, np.full(4, 0.25))


def test_topk_ties_partial():
    lg = np.zeros(16)
    lg[[9, 3, 12, 5, 7]] = 2.0  # five tied maxima: lowest four indices win
    ids, p, _ = oracle.topk_softmax(lg, 4)
    assert ids.tolist() == [3, 5, 7, 9]
    assert np.array_equal(p, np.full(4, 0.25))


def test_topk_log_weights_closed_form():
    lg = np.full(64, -30.0)
    lg[[40, 2, 17, 63]] = np.log([4.0, 3.0, 2.0, 1.0])
    ids, p, _ = oracle.topk_softmax(lg, 4)
    assert ids.tolist() == [40, 2, 17, 63]
    assert np.allclose(p, [0.4, 0.3, 0.2, 0.1], rtol=1e-15)


def test_topk_weights_sum_to_one_and_follow_logit_order():
    r = rng(8)
    for _ in range(50):
        lg = r.normal(size=512) * r.uniform(0.1, 10)
        ids, p, _ = oracle.topk_softmax(lg, 4)
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(np.diff(lg[ids]) <= 0) and np.all(np.diff(p) <= 0)
        assert set(ids.tolist()) == set(np.argsort(-lg, kind="stable")[:4].tolist())


def test_topk_one_selects_the_maximum_with_weight_one():
    lg = np.linspace(-1, 1, 64)[::-1].copy()
    lg[37] = 5.0
    ids, p, _ = oracle.topk_softmax(lg, 1)
    assert ids.tolist() == [37] and p.tolist() == [1.0]


def test_topk_of_every_logit_is_the_full_softmax_in_descending_order():
    # k = E: every expert selected; the weights are the softmax over all of
    # them, listed from the largest logit down (ties: lower index first)
    lg = np.array([0.5, 2.0, -1.0, 2.0, 0.0])
    ids, p, _ = oracle.topk_softmax(lg, 5)
    assert ids.tolist() == [1, 3, 0, 4, 2]
    e = np.exp(lg - lg.max())
    assert np.allclose(p, (e / e.sum())[[1, 3, 0, 4, 2]], rtol=1e-15)


def test_topk_nan_is_never_selected_and_is_reported():
    lg = np.linspace(1, 0, 16)
    lg[0] = np.nan
    lg[5] = np.nan
    ids, p, nan = oracle.topk_softmax(lg, 4)
    assert nan and ids.tolist() == [1, 2, 3, 4]


def test_topk_with_fewer_numbers_than_k_gives_nan_weight_zero():
    """NaN ranks below every number (the reading: NaN as -inf): with three
    numbers among six logits, top-4 takes the three numbers in order and
    then the lowest-index NaN, whose weight is exp(-inf) = 0; the numbers'
    weights are the softmax of the three."""
    lg = np.array([np.nan, 1.0, np.nan, 0.5, np.nan, 2.0])
    ids, p, nan = oracle.topk_softmax(lg, 4)
    assert nan and ids.tolist() == [5, 1, 3, 0]
    e = np.exp(np.array([2.0, 1.0, 0.5]) - 2.0)
    assert np.allclose(p[:3], e / e.sum(), rtol=1e-15) and p[3] == 0.0


# ------------------------------------------------------- SwiGLU / sigmoid ----

def test_sigmoid_and_swiglu_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert abs(oracle.sigmoid(math.log(3)) - 0.75) < 1e-15
    assert abs(oracle.sigmoid(-1.7) + oracle.sigmoid(1.7) - 1.0) < 1e-15
    assert oracle.swiglu(0.0, 5.0) == 0.0
    assert abs(oracle.swiglu(math.log(3), 2.0) - 0.75 * math.log(3) * 2.0) < 1e-15
    assert abs(oracle.swiglu(40.0, 1.5) / (40.0 * 1.5) - 1.0) < 1e-15  # silu(g)/g -> 1
    assert abs(oracle.swiglu(-40.0, 1.5)) < 1e-15


# ------------------------------------------------------------ one expert ----

def _const_expert(H, I, G, gate, up, down):
    """Expert whose three matrices have constant code/scale/bias each:
    gate/up/down = (code, scale_bits, bias_bits)."""
    n, ng = H * I, H * I // G
    q = np.concatenate([np.full(n, gate[0]), np.full(n, up[0]), np.full(n, down[0])]).astype(np.uint8)
    s = np.concatenate([np.full(ng, gate[1]), np.full(ng, up[1]), np.full(ng, down[1])]).astype(np.uint16)
    b = np.concatenate([np.full(ng, gate[2]), np.full(ng, up[2]), np.full(ng, down[2])]).astype(np.uint16)
    return synth.ExpertLogical(4, q, s, b)


def test_expert_ffn_closed_form():
    H, I, G = 128, 64, 64
    # gate weight = 3 * 2^-7 everywhere, up weight = 2^-5 + (-2^-6), down weight = 1
    ex = _const_expert(H, I, G, (3, bf16_pow2(-7), 0), (1, bf16_pow2(-5), 0xBC80), (1, BF16_ONE, 0))
    x = np.full(H, 0.5)
    out = oracle.expert_ffn(ex, H, I, G, x)
    g = 3 * 2.0 ** -7 * 0.5 * H
    u = (2.0 ** -5 - 2.0 ** -6) * 0.5 * H
    a = g / (1 + math.exp(-g)) * u
    assert np.allclose(out["g"], g, rtol=1e-15) and np.allclose(out["u"], u, rtol=1e-15)
    assert np.allclose(out["a"], a, rtol=1e-14)
    assert np.allclose(out["y"], I * a, rtol=1e-14)


def test_expert_ffn_uses_transposed_down_shape():
    """gate/up are [I][H], down is [H][I] (H != I): a one-hot pattern in each
    matrix must land on the right output."""
    H, I, G = 128, 64, 64
    n, ng = H * I, H * I // G
    q = np.zeros(3 * n, np.uint8)
    s = np.full(3 * ng, BF16_ONE, np.uint16)
    b = np.zeros(3 * ng, np.uint16)
    q[0 * n + 5 * H + 70] = 2      # gate row 5, input 70
    q[1 * n + 5 * H + 70] = 3      # up row 5, input 70
    q[2 * n + 100 * I + 5] = 1     # down row 100, input 5
    ex = synth.ExpertLogical(4, q, s, b)
    x = np.zeros(H)
    x[70] = 1.0
    out = oracle.expert_ffn(ex, H, I, G, x)
    a5 = 2.0 / (1 + math.exp(-2.0)) * 3.0
    assert out["a"][5] == pytest.approx(a5, rel=1e-15)
    assert np.count_nonzero(out["a"]) == 1
    assert out["y"][100] == pytest.approx(a5, rel=1e-15) and np.count_nonzero(out["y"]) == 1


# ------------------------------------------------------ combine + norm ----

def test_rmsnorm_of_constant_residual():
    H = 256
    w = synth.norm_weight(synth.TINY, 0)
    for c in (1.0, -3.5, 1e-4):
        y = np.zeros((5, H))
        h_out, xn, _, _ = oracle.combine_rmsnorm(y, np.full(4, 0.25), 0.5, np.full(H, c), w, 1e-6)
        assert np.array_equal(h_out, np.full(H, c))
        assert np.allclose(xn, w.astype(np.float64) * c / math.sqrt(c * c + 1e-6), rtol=1e-15)


def test_combine_weights_gate_and_residual():
    H = 64
    r = rng(9)
    y = r.normal(size=(5, H))
    p = np.array([0.4, 0.3, 0.2, 0.1])
    h = r.normal(size=H)
    h_out, xn, _, _ = oracle.combine_rmsnorm(y, p, 0.25, h, np.ones(H, np.float32), 0.0)
    expect = h + 0.4 * y[0] + 0.3 * y[1] + 0.2 * y[2] + 0.1 * y[3] + 0.25 * y[4]
    assert np.allclose(h_out, expect, rtol=1e-15, atol=1e-15)
    assert abs(np.mean(xn ** 2) - 1.0) < 1e-13  # RMS 1 with unit weight and eps 0


# -------------------------------------------------------------- one layer ----

def _tiny_layer(wl, layer=0):
    lw = oracle.LayerWeights(synth.router(wl, layer), synth.shared_gate(wl, layer), synth.norm_weight(wl, layer), {})
    for s, ex in enumerate(synth.experts(wl, layer, range(wl.n_experts + 1))):
        lw.experts[s] = ex
    return lw


def test_layer_invariant_under_expert_relabelling():
    wl = synth.TINY
    lw = _tiny_layer(wl)
    x = synth.tokens(wl, 1)[0].astype(np.float64)
    base = oracle.layer_token(wl, lw, x, x)
    perm = rng(10).permutation(wl.n_experts)  # new slot j holds old expert perm[j]
    lw2 = oracle.LayerWeights(lw.w_router[perm], lw.w_shared_gate, lw.norm_w,
                              {j: lw.experts[int(perm[j])] for j in range(wl.n_experts)})
    lw2.experts[wl.n_experts] = lw.experts[wl.n_experts]
    out = oracle.layer_token(wl, lw2, x, x)
    assert perm[out["ids"]].tolist() == base["ids"].tolist()
    assert np.allclose(out["h"], base["h"], rtol=1e-14, atol=1e-14)
    assert np.allclose(out["xn"], base["xn"], rtol=1e-14, atol=1e-14)


def test_layer_with_identical_experts_reduces_to_one_expert():
    """All routed experts equal: sum_k p_k y = y (weights sum to one)."""
    wl = synth.TINY
    lw = _tiny_layer(wl)
    same = lw.experts[7]
    for s in range(wl.n_experts):
        lw.experts[s] = same
    x = synth.tokens(wl, 1, stream=3)[0].astype(np.float64)
    h = synth.tokens(wl, 1, stream=4)[0].astype(np.float64)  # residual differs from the normed input
    out = oracle.layer_token(wl, lw, h, x)
    one = oracle.expert_ffn(same, wl.hidden, wl.inter, 64, x)
    sh = oracle.expert_ffn(lw.experts[wl.n_experts], wl.hidden, wl.inter, 64, x)
    z = float(lw.w_shared_gate.astype(np.float64) @ x)
    gamma = 1.0 / (1.0 + math.exp(-z))
    h_expect = h + one["y"] + gamma * sh["y"]
    assert out["gamma"] == pytest.approx(gamma, rel=1e-14)
    assert np.allclose(out["h"], h_expect, rtol=1e-12, atol=1e-12)


def test_layer_logits_given_routes_on_them():
    wl = synth.TINY
    lw = _tiny_layer(wl)
    x = synth.tokens(wl, 1)[0].astype(np.float64)
    lg = np.full(wl.n_experts, -5.0, np.float32)
    lg[[11, 4, 9, 0]] = [3.0, 2.0, 1.0, 0.0]
    out = oracle.layer_token(wl, lw, x, x, logits_in=lg)
    assert out["ids"].tolist() == [11, 4, 9, 0]


def test_layer_residual_enters_only_the_sum():
    """The router, the shared gate and every expert read the normed input xn
    only; the residual stream h is added to their combined output.  So with
    xn fixed, moving h changes nothing but h', by exactly the move."""
    wl = synth.TINY
    lw = _tiny_layer(wl)
    x = synth.tokens(wl, 1, stream=7)[0].astype(np.float64)
    h1 = synth.tokens(wl, 1, stream=8)[0].astype(np.float64) * 4
    h2 = -3 * h1 + 1.0
    a = oracle.layer_token(wl, lw, h1, x)
    b = oracle.layer_token(wl, lw, h2, x)
    assert a["ids"].tolist() == b["ids"].tolist()
    for key in ("logits", "p", "gamma", "y"):
        assert np.array_equal(a[key], b[key]), key
    moved = b["h"] - a["h"]
    assert np.allclose(moved, h2 - h1, rtol=1e-13, atol=1e-13 * np.abs(h1).max())
    # and the router reads xn: the same h with another xn routes differently
    c = oracle.layer_token(wl, lw, h1, x[::-1].copy())
    assert not np.array_equal(a["logits"], c["logits"])


# -------------------------------------------------- quantiser round trip ----

@pytest.mark.parametrize("bits", [4, 2])
def test_quantise_dequantise_round_trip_exact(bits):
    r = rng(11 + bits)
    rows, cols, G = 4, 256, 64
    qmax = (1 << bits) - 1
    q = r.integers(0, qmax + 1, size=(rows, cols), dtype=np.uint8)
    q[:, ::G] = 0          # every group holds both extremes
    q[:, 1::G] = qmax
    s = synth.f32_to_bf16(r.uniform(0.005, 0.08, size=(rows, cols // G)).astype(np.float32))
    b = synth.f32_to_bf16((-8 * synth.bf16_to_f32(s)).astype(np.float32))
    w = oracle.dequantize(q, s, b, G)
    q2, s2, b2 = oracle.quantize(w.ravel(), G, bits)
    assert np.array_equal(q2.reshape(rows, cols), q)
    assert np.array_equal(s2, synth.bf16_to_f32(s).astype(np.float64).ravel())
    assert np.array_equal(b2, synth.bf16_to_f32(b).astype(np.float64).ravel())


def test_quantiser_error_at_most_half_step():
    w = rng(12).normal(size=64 * 40)
    for bits in (4, 2):
        q, s, b = oracle.quantize(w, 64, bits)
        back = q.astype(np.float64) * np.repeat(s, 64) + np.repeat(b, 64)
        assert np.all(np.abs(back - w) <= np.repeat(s, 64) / 2 * (1 + 1e-12))


@pytest.mark.parametrize("bits", [4, 2])
def test_stored_format_quantiser_recovers_exact_inputs(bits):
    """Weights that are q * S + B with bf16 S, B (each group holding both
    code extremes) come back as exactly q, S, B from the fp32 quantiser."""
    r = rng(21 + bits)
    G, n_groups = 64, 48
    qmax = (1 << bits) - 1
    q = r.integers(0, qmax + 1, size=(n_groups, G), dtype=np.uint8)
    q[:, 0], q[:, 1] = 0, qmax
    # S and B chosen so that every q * S + B is exact in fp32 and (hi - lo) / qmax == S exactly
    S = synth.f32_to_bf16((2.0 ** r.integers(-9, -3, size=n_groups)).astype(np.float32))
    B = synth.f32_to_bf16((-(2.0 ** r.integers(-6, 0, size=n_groups)) * r.integers(1, 4, size=n_groups)).astype(np.float32))
    Sf, Bf = synth.bf16_to_f32(S), synth.bf16_to_f32(B)
    w = (q.astype(np.float32) * Sf[:, None] + Bf[:, None]).astype(np.float32)
    assert np.array_equal(w.astype(np.float64), q * Sf[:, None].astype(np.float64) + Bf[:, None])  # exact
    q2, s2, b2 = oracle.quantize_f32(w, G, bits)
    assert np.array_equal(q2.reshape(n_groups, G), q)
    assert np.array_equal(s2, S) and np.array_equal(b2, B)


def test_stored_format_quantiser_error_bound_and_special_groups():
    """Round-trip error of the fp32 quantiser: at most S/2, plus what the
    bf16 rounding of the scale (qmax of its half-ulp) and of the bias can
    add; a constant group gives scale 0 and codes 0; negative and positive
    groups alike."""
    r = rng(22)
    for bits in (4, 2):
        qmax = (1 << bits) - 1
        w = np.concatenate([r.normal(size=64 * 30), r.normal(loc=5.0, size=64 * 5), -r.uniform(1, 3, 64 * 5),
                            np.full(64, 0.375)]).astype(np.float32)
        q, s, b = oracle.quantize_f32(w, 64, bits)
        S, B = synth.bf16_to_f32(s).astype(np.float64), synth.bf16_to_f32(b).astype(np.float64)
        back = q.astype(np.float64) * np.repeat(S, 64) + np.repeat(B, 64)
        lo = w.reshape(-1, 64).min(axis=1).astype(np.float64)
        bound = S / 2 + qmax * S * 2.0 ** -8 + np.abs(lo) * 2.0 ** -8 + 1e-12
        assert np.all(np.abs(back - w).reshape(-1, 64) <= bound[:, None])
        assert s[-1] == 0 and np.all(q[-64:] == 0) and synth.bf16_to_f32(b[-1:])[0] == np.float32(0.375)
        assert q.max() <= qmax


def test_stored_format_quantiser_rounds_bf16_to_nearest_even():
    """The stored scale and bias are the nearest bf16 values, ties to the
    even significand (bf16 keeps 8 significant bits: 1 + 2^-8 lies halfway
    between 1 and 1 + 2^-7).  Groups of 64 built so that the fp32 minimum and
    the fp32 scale (hi - lo) / 15 are exactly such halfway values."""
    G = 64

    def group(lo, span):
        g = np.linspace(0.0, 1.0, G).astype(np.float32) * np.float32(span) + np.float32(lo)
        g[0], g[-1] = lo, np.float32(lo) + np.float32(span)
        return g

    cases = [  # (minimum, hi - lo, expected bias bits, expected scale bits)
        (1 + 2.0 ** -8, 15 * (1 + 2.0 ** -8), 0x3F80, 0x3F80),       # ties down to even
        (1 + 3 * 2.0 ** -8, 15 * (1 + 3 * 2.0 ** -8), 0x3F82, 0x3F82),  # ties up to even
        (-(1 + 2.0 ** -8), 15 * 0.5, 0xBF80, 0x3F00),                # negative tie, exact scale
        (1 + 2.0 ** -8 + 2.0 ** -20, 15 * (1 + 2.0 ** -8 + 2.0 ** -20), 0x3F81, 0x3F81),  # above the tie
    ]
    w = np.concatenate([group(lo, span) for lo, span, _, _ in cases])
    for (lo, span, _, _), g in zip(cases, w.reshape(-1, G)):
        assert g.min() == np.float32(lo) and np.float32(g.max() - g.min()) / np.float32(15) == np.float32(span / 15)
    _, s, b = oracle.quantize_f32(w, G, 4)
    assert [int(v) for v in b] == [c[2] for c in cases]
    assert [int(v) for v in s] == [c[3] for c in cases]


@pytest.mark.parametrize("bits", [4, 2])
def test_stored_format_quantiser_picks_the_nearest_stored_grid_point(bits):
    """Each code selects, among the points c * S + B (c = 0 .. 2^bits - 1) of
    the STORED bf16 scale S and bias B, the one nearest the weight, up to the
    fp32 rounding of (w - B) / S: codes taken from the unrounded scale or
    minimum miss it by up to a few hundredths of S."""
    r = rng(23 + bits)
    qmax = (1 << bits) - 1
    w = np.concatenate([r.normal(size=64 * 60), r.normal(loc=-3.0, scale=0.2, size=64 * 20)]).astype(np.float32)
    q, s, b = oracle.quantize_f32(w, 64, bits)
    S = np.repeat(synth.bf16_to_f32(s).astype(np.float64), 64)
    B = np.repeat(synth.bf16_to_f32(b).astype(np.float64), 64)
    grid = np.arange(qmax + 1)[None, :] * S[:, None] + B[:, None]
    best = np.abs(grid - w.astype(np.float64)[:, None]).min(axis=1)
    got = np.abs(q.astype(np.float64) * S + B - w)
    assert np.all(got <= best + 1e-5 * S)


def test_stored_format_quantiser_stores_a_negative_zero_minimum_as_plus_zero():
    """A group whose minimum is -0 stores bias +0 (bits 0), the reading the
    oracle states; its codes are those of the +0 minimum."""
    g = np.linspace(0.0, 1.5, 64).astype(np.float32)
    g[0] = -0.0
    q, s, b = oracle.quantize_f32(g, 64, 4)
    g2 = g.copy()
    g2[0] = 0.0
    q2, s2, b2 = oracle.quantize_f32(g2, 64, 4)
    assert int(b[0]) == 0 and int(b2[0]) == 0
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


# ------------------------------------------------------------ byte counts ----

def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split("=")
            vals[k.strip()] = float(v)
    return vals


def test_expert_record_size_matches_pages():
    """3 matrices of hidden x 1024 codes at 4 bits plus one bf16 scale and
    bias per 64 codes is 6.75 MiB, the pages' per-expert figure."""
    g = _golden()
    H, I, G = int(g["hidden"]), 1024, 64
    int4 = 3 * H * I // 2 + 3 * H * I // G * 4
    int2 = 3 * H * I // 4 + 3 * H * I // G * 4
    assert int4 == 7_077_888 and int4 / 2 ** 20 == g["expert_mb_int4"]
    assert int2 / 2 ** 20 == 3.75
    # only the routed experts change precision between the 4-bit and 2-bit
    # models: 60 layers x 512 experts x 3 MiB = 90 GiB, vs 209 - 120 = 89
    # (each printed figure rounded to 1 GB)
    delta = g["layers"] * g["experts_per_layer"] * (int4 - int2) / 2 ** 30
    assert abs(delta - (g["model_gb_int4"] - g["model_gb_int2"])) <= 1.0


# ------------------------------------------------------------ error scales ----
# The oracle's error scale S of an output is a first-order bound: if every
# input of a step moves by at most eps times its own scale (and every term of
# a sum by eps times its magnitude), the output moves by at most eps * S, and
# some choice of signs reaches it.  Each pin below moves the inputs of one
# step by +-eps * S and measures the response of the oracle's own value
# function (finite differences in fp64), so the scale is tied to how the
# output actually depends on its inputs, not to a retyped formula.

EPS = 1e-7


def _tiny_expert(seed, H=256, I=128):
    wl = synth.Workload(hidden=H, inter=I, n_experts=4)
    return wl, synth.expert(wl, seed % 7, seed % 4)


def _dense(q, s, b, G):
    return oracle.dequantize(q, s, b, G)


def test_error_scale_of_router_and_qgemv_is_sum_of_absolute_terms():
    """S of a dense or dequantised product is sum_j |w_j x_j|: moving every
    x_j by eps |x_j| sign(w_j) moves y by exactly eps * S."""
    r = rng(40)
    W = r.normal(0, 0.02, size=(9, 192)).astype(np.float32)
    x = r.normal(size=192)
    y, S = oracle.gemv_f32(W, x)
    for i in range(9):
        d = EPS * np.abs(x) * np.sign(W[i].astype(np.float64))
        yp, _ = oracle.gemv_f32(W, x + d)
        assert (yp[i] - y[i]) / EPS == pytest.approx(S[i], rel=1e-6)
    wl, ex = _tiny_expert(1)
    n = wl.hidden * wl.inter
    q, s, b = ex.q[:n].reshape(wl.inter, wl.hidden), ex.scale[:n // 64].reshape(wl.inter, -1), \
        ex.bias[:n // 64].reshape(wl.inter, -1)
    w = _dense(q, s, b, 64)
    xq = synth.tokens(wl, 1, stream=3)[0].astype(np.float64)
    yq, Sq = oracle.qgemv(q, s, b, 64, xq)
    for i in (0, 17, wl.inter - 1):
        d = EPS * np.abs(xq) * np.sign(w[i])
        yp, _ = oracle.qgemv(q, s, b, 64, xq + d)
        assert (yp[i] - yq[i]) / EPS == pytest.approx(Sq[i], rel=1e-6)


def test_error_scale_of_swiglu_outputs():
    """S_a: the worst of the four sign choices of (g +- eps S_g, u +- eps S_u)
    moves silu(g) u by eps S_a, to first order.  A wrong derivative of silu
    (a dropped g sigmoid'(g) term, a swapped S_g / S_u) fails here."""
    for seed in range(3):
        wl, ex = _tiny_expert(seed)
        x = synth.tokens(wl, 1, stream=10 + seed)[0].astype(np.float64) * (1 + 2 * seed)
        out = oracle.expert_ffn(ex, wl.hidden, wl.inter, 64, x)
        g, u, a = out["g"], out["u"], out["a"]
        for i in range(wl.inter):
            resp = max(abs(oracle.swiglu(g[i] + sg * EPS * out["S_g"][i], u[i] + su * EPS * out["S_u"][i]) - a[i])
                       for sg in (-1, 1) for su in (-1, 1)) / EPS
            assert resp == pytest.approx(out["S_a"][i], rel=1e-4, abs=1e-12), (seed, i)


def test_error_scale_of_down_products_propagates_through_down_rows():
    """S_y of an expert output = its own terms sum_j |Wd_rj a_j| plus
    sum_j |Wd_rj| S_a,j.  The second part is measured: moving each a_j by
    eps S_a,j sign(Wd_rj) moves y_r by eps times it.  H != I, so summing the
    down matrix along the wrong axis cannot pass."""
    wl, ex = _tiny_expert(2)
    H, I = wl.hidden, wl.inter
    x = synth.tokens(wl, 1, stream=20)[0].astype(np.float64)
    out = oracle.expert_ffn(ex, H, I, 64, x)
    n = H * I
    qd = ex.q[2 * n:].reshape(H, I)
    sd = ex.scale[2 * n // 64:].reshape(H, I // 64)
    bd = ex.bias[2 * n // 64:].reshape(H, I // 64)
    wd = _dense(qd, sd, bd, 64)
    y0, own = oracle.qgemv(qd, sd, bd, 64, out["a"])
    assert np.array_equal(y0, out["y"])
    for r in range(0, H, 5):
        yp, _ = oracle.qgemv(qd, sd, bd, 64, out["a"] + EPS * out["S_a"] * np.sign(wd[r]))
        prop = (yp[r] - y0[r]) / EPS
        assert out["S_y"][r] - own[r] == pytest.approx(prop, rel=1e-5), r


def test_error_scale_of_shared_gate():
    """S_gamma = d sigmoid / dz * S_z: z +- eps S_z moves gamma by eps S_gamma."""
    wl = synth.TINY
    lw = _tiny_layer(wl)
    x = synth.tokens(wl, 1, stream=4)[0].astype(np.float64) * 3
    ref = oracle.layer_token(wl, lw, x, x)
    z, Sz = oracle.gemv_f32(lw.w_shared_gate[None], x)
    resp = max(abs(oracle.sigmoid(z[0] + sgn * EPS * Sz[0]) - ref["gamma"]) for sgn in (-1, 1)) / EPS
    assert resp == pytest.approx(ref["S_gamma"], rel=1e-5)


def test_error_scale_of_combine():
    """S_h - 1e-2 (the 1e-2 carries the inputs' absolute 1e-5 slack) is the
    response of h' when h moves by eps |h|, every y_k by eps (|y_k| + S_y,k)
    and gamma by eps S_gamma towards the sign of y_s: the sum's own terms plus
    its inputs' errors, each with its weight (p_k >= 0, gamma >= 0)."""
    r = rng(41)
    H, k = 64, 4
    y = r.normal(size=(k + 1, H)) * 2
    S_y = np.abs(r.normal(size=(k + 1, H))) * 5
    p = r.dirichlet(np.ones(k))
    gamma, S_gamma = 0.3, 0.7
    h = r.normal(size=H)
    w = (1 + 0.1 * r.normal(size=H)).astype(np.float32)
    ho, _, Sh, _ = oracle.combine_rmsnorm(y, p, gamma, h, w, 1e-6, S_y=S_y, S_gamma=S_gamma)
    for sgn in (1.0, -1.0):
        rows = np.sign(y[k]) == sgn
        yp = y + EPS * (np.abs(y) + S_y)
        hp, _, _, _ = oracle.combine_rmsnorm(yp, p, gamma + sgn * EPS * S_gamma, h + EPS * np.abs(h), w, 1e-6,
                                             S_y=S_y, S_gamma=S_gamma)
        resp = (hp - ho) / EPS
        assert np.allclose(resp[rows], Sh[rows] - 1e-2, rtol=1e-5, atol=1e-9)


def test_error_scale_of_rmsnorm():
    """S_xn - 1e-3 |xn'| bounds the response of xn'_i to moves of h' by at
    most eps S_h, and the worst-case move (h'_i towards w_i, every other h'_j
    against the sign of h'_i h'_j w_i, which moves r the same way) reaches it
    up to the cross term of h'_i with itself, 2 |w_i| h'_i^2 r^3 S_h,i / H.
    A missing r-error term, or one without its 1/H, fails here."""
    r_ = rng(42)
    H = 64
    h = r_.normal(size=H) * 1.5
    w = (1 + 0.1 * r_.normal(size=H)).astype(np.float32)
    z = np.zeros((2, H))
    # k = 1, zero expert outputs and gamma 0: h' = h, S_h = |h| + 1e-2
    ho, xo, Sh, Sx = oracle.combine_rmsnorm(z, np.ones(1), 0.0, h, w, 1e-6)
    assert np.array_equal(ho, h)
    rr = 1.0 / math.sqrt(np.mean(h * h) + 1e-6)
    bound = Sx - 1e-3 * np.abs(xo)
    for i in range(H):
        wi = float(w[i])
        d = -EPS * Sh * np.sign(h) * np.sign(wi * h[i])
        d[i] = EPS * Sh[i] * np.sign(wi)
        _, xp, _, _ = oracle.combine_rmsnorm(z, np.ones(1), 0.0, h + d, w, 1e-6)
        resp = abs(xp[i] - xo[i]) / EPS
        cross = 2 * abs(wi) * h[i] ** 2 * rr ** 3 * Sh[i] / H
        assert resp <= bound[i] * (1 + 1e-5), i
        assert resp >= (bound[i] - cross) * (1 - 1e-5) - 1e-9, i
    # random moves within the scales never exceed the bound
    for t in range(20):
        d = EPS * Sh * r_.uniform(-1, 1, size=H)
        _, xp, _, _ = oracle.combine_rmsnorm(z, np.ones(1), 0.0, h + d, w, 1e-6)
        assert np.all(np.abs(xp - xo) <= EPS * bound * (1 + 1e-5))


def test_layer_error_scales_compose_the_steps():
    """oracle_layer_token's scales are those of its steps chained: S_y of each
    selected expert from expert_ffn, then S_h / S_xn from combine_rmsnorm with
    those S_y and S_gamma."""
    wl = synth.TINY
    lw = _tiny_layer(wl)
    x = synth.tokens(wl, 1, stream=6)[0].astype(np.float64)
    ref = oracle.layer_token(wl, lw, x, x)
    for j, slot in enumerate(list(ref["ids"]) + [wl.n_experts]):
        e = oracle.expert_ffn(lw.experts[int(slot)], wl.hidden, wl.inter, 64, x)
        assert np.array_equal(e["S_y"], ref["S_y"][j])
    _, _, Sh, Sx = oracle.combine_rmsnorm(ref["y"], ref["p"], ref["gamma"], x, lw.norm_w, wl.eps,
                                          S_y=ref["S_y"], S_gamma=ref["S_gamma"])
    assert np.array_equal(Sh, ref["S_h"]) and np.array_equal(Sx, ref["S_xn"])


def test_openmp_timing_build_computes_the_same_values():
    """The OpenMP build that the CPU baseline times (output rows over
    threads) gives the plain build's values bit for bit: the rows are
    independent, each summed in the same order."""
    wl = synth.TINY
    lw = oracle.LayerWeights(synth.router(wl, 0), synth.shared_gate(wl, 0), synth.norm_weight(wl, 0),
                             dict(zip(range(wl.n_experts + 1), synth.experts(wl, 0, range(wl.n_experts + 1)))))
    x = synth.tokens(wl, 3, stream=5).astype(np.float64)
    keys = ("h", "xn", "S_h", "S_xn", "p", "gamma")
    try:
        oracle.set_threads(1)
        plain = [oracle.layer_token(wl, lw, x[t], x[t]) for t in range(3)]
        oracle.set_threads(4)
        omp = [oracle.layer_token(wl, lw, x[t], x[t]) for t in range(3)]
    finally:
        oracle.set_threads(1)
    for a, b in zip(plain, omp):
        assert a["ids"].tolist() == b["ids"].tolist()
        for k in keys:
            assert np.array_equal(np.asarray(a[k]), np.asarray(b[k])), k
