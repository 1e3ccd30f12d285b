"""The seeded input generator: known answers and distribution checks."""
import numpy as np
import torch

import synth


def test_splitmix64_known_answer():
    """Element i of a stream with key K is the (i+1)-th SplitMix64 output for
    state K; the reference sequence for state 1234567 is widely published."""
    assert synth.words(1234567, 0, 5).tolist() == [
        6457827717110365317, 3203168211198807973, 9817491932198370423,
        4593380528125082431, 16408922859458223821]


def test_streams_are_random_access():
    k = synth.key(0, synth.K_CODES[0], 3, 17)
    full = synth.codes(k, 4, 1000)
    assert np.array_equal(synth.codes(k, 4, 301, first=77), full[77:378])
    w = synth.words(k, 10, 5)
    assert np.array_equal(w, synth.words(k, 0, 15)[10:])


def test_code_distribution_uniform():
    for bits in (4, 2):
        c = synth.codes(synth.key(0, 1, 0, 0), bits, 1 << 20)
        n = 1 << bits
        assert c.max() == n - 1 and c.min() == 0
        hist = np.bincount(c, minlength=n)
        expect = c.size / n
        chi2 = ((hist - expect) ** 2 / expect).sum()
        assert chi2 < 50  # df = 15 or 3


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).normal(size=10000).astype(np.float32) * 3
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0]  # ties to even
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16(x), ref)


def test_expert_value_ranges():
    wl = synth.TINY
    ex = synth.expert(wl, 0, 2)
    s = synth.bf16_to_f32(ex.scale)
    b = synth.bf16_to_f32(ex.bias)
    assert s.min() >= 0.005 * (1 - 2 ** -8) and s.max() <= 0.02 * (1 + 2 ** -8)
    noise = b + 8 * s
    assert abs(noise.mean()) < 2e-4 and 0.5e-3 < noise.std() < 1.5e-3
    ex2 = synth.expert(synth.Workload(hidden=256, inter=128, n_experts=16, bits=2), 0, 2)
    assert ex2.q.max() == 3
    s2 = synth.bf16_to_f32(ex2.scale)
    assert s2.min() >= 0.02 * (1 - 2 ** -8) and s2.max() <= 0.08 * (1 + 2 ** -8)
    assert np.array_equal(ex2.bias, synth.f32_to_bf16(-1.5 * s2))


def test_shared_expert_keeps_four_bits_in_two_bit_layers():
    wl = synth.Workload(hidden=256, inter=128, n_experts=16, bits=2)
    assert synth.expert(wl, 0, wl.n_experts).q.max() == 15


def test_normals():
    x = synth.normal_f32(synth.key(0, synth.K_X, 0, 0), 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    w = synth.norm_weight(synth.LAYER, 0)
    assert abs(w.mean() - 1) < 0.01 and abs(w.std() - 0.1) < 0.01


def test_zipf_gumbel_sampling_follows_one_over_rank():
    wl = synth.LAYER
    counts = np.zeros(wl.n_experts)
    first = np.zeros(wl.n_experts)
    steps = 40
    for step in range(steps):
        lg, r2i = synth.zipf_gumbel_logits(wl, step, 64)
        top = np.argsort(-lg, axis=1, kind="stable")[:, :4]
        for t in range(64):
            counts[top[t]] += 1
            first[top[t, 0]] += 1
    # rank -> id permutation is fixed per seed; the top-1 draw is exactly
    # categorical with p_r = (1/r) / H_512
    H512 = (1.0 / np.arange(1, 513)).sum()
    n = steps * 64
    for r in range(3):
        p = 1.0 / (r + 1) / H512
        assert abs(first[r2i[r]] / n - p) < 4 * np.sqrt(p * (1 - p) / n)
    assert counts.sum() == n * 4
