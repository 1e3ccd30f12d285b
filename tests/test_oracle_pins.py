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


def test_topk_nan_is_never_selected_and_is_reported():
    lg = np.linspace(1, 0, 16)
    lg[0] = np.nan
    lg[5] = np.nan
    ids, p, nan = oracle.topk_softmax(lg, 4)
    assert nan and ids.tolist() == [1, 2, 3, 4]


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
