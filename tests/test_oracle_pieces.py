"""Pins of the oracle's textbook pieces against torch CPU routines and closed forms.

Each piece is checked against an independent definition (a library routine or
a mathematical identity), never against a retyped copy of its own formula.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(123)


def test_rmsnorm_matches_torch():
    x = rng.standard_normal(96)
    g = 1 + 0.3 * rng.standard_normal(96)
    got = oracle.rmsnorm(x, g, 1e-6)
    ref = F.rms_norm(torch.tensor(x), (96,), torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-15)
    # the output of a gain-1 norm has mean square 1 (up to eps)
    y = oracle.rmsnorm(x, np.ones(96), 0.0)
    assert abs(np.mean(y * y) - 1) < 1e-13


def test_linear_matches_matmul():
    W = rng.standard_normal((7, 5))
    x = rng.standard_normal(5)
    np.testing.assert_allclose(oracle.linear(W, x), W @ x, rtol=1e-13)


def test_activations_match_torch_and_closed_forms():
    xs = np.linspace(-6, 6, 49)
    t = torch.tensor(xs)
    gelu = np.array([oracle.scalar("gelu", x) for x in xs])
    silu = np.array([oracle.scalar("silu", x) for x in xs])
    sig = np.array([oracle.scalar("sigmoid", x) for x in xs])
    np.testing.assert_allclose(gelu, F.gelu(t).numpy(), rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(silu, F.silu(t).numpy(), rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(sig, torch.sigmoid(t).numpy(), rtol=1e-13, atol=1e-16)
    with open(os.path.join(GOLDEN, "activations.json")) as f:
        gold = json.load(f)
    for name, pairs in gold["values"].items():
        for x, y in pairs:
            assert abs(oracle.scalar(name, x) - y) < 1e-15, (name, x)


def _rope_complex(v, pos, theta):
    """Rotation written as complex multiplication z_i * exp(i pos theta^(-2i/dh))."""
    dh = v.shape[0]
    half = dh // 2
    z = v[:half] + 1j * v[half:]
    k = np.arange(half)
    z = z * np.exp(1j * pos * theta ** (-2.0 * k / dh))
    return np.concatenate([z.real, z.imag])


@pytest.mark.parametrize("dh", [16, 64, 128])
def test_rope_complex_form_and_invariants(dh):
    v = rng.standard_normal(dh)
    for pos in (0, 1, 7, 1023, 4095):
        got = oracle.rope(v, pos)
        np.testing.assert_allclose(got, _rope_complex(v, pos, 1e4), rtol=0, atol=1e-12)
        assert abs(np.linalg.norm(got) - np.linalg.norm(v)) < 1e-12
    np.testing.assert_array_equal(oracle.rope(v, 0), v)
    # scores depend only on the relative offset of the two positions
    q, k = rng.standard_normal(dh), rng.standard_normal(dh)
    a = oracle.rope(q, 40) @ oracle.rope(k, 33)
    b = oracle.rope(q, 1007) @ oracle.rope(k, 1000)
    assert abs(a - b) < 1e-10


@pytest.mark.parametrize("n", [1, 2, 9, 130])
def test_attend_matches_sdpa(n):
    dh = 16
    q = rng.standard_normal(dh)
    K = rng.standard_normal((n, dh))
    V = rng.standard_normal((n, dh))
    got = oracle.attend(q, K, V)
    ref = F.scaled_dot_product_attention(
        torch.tensor(q)[None, None, None], torch.tensor(K)[None, None],
        torch.tensor(V)[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_attend_special_cases():
    dh = 8
    V = rng.standard_normal((5, dh))
    # one key: output is that value exactly
    np.testing.assert_array_equal(oracle.attend(rng.standard_normal(dh), V[:1], V[:1]), V[0])
    # zero query: uniform average of the values
    np.testing.assert_allclose(oracle.attend(np.zeros(dh), rng.standard_normal((5, dh)), V),
                               V.mean(0), rtol=1e-13)
    # huge scores do not overflow (max subtraction)
    q = np.full(dh, 100.0)
    K = np.zeros((5, dh)); K[3] = 10.0
    np.testing.assert_allclose(oracle.attend(q, K, V), V[3], rtol=1e-13)


# ---------------------------------------------------------- serving loop
def test_lm_head_is_embedding_matmul():
    """Next-token logits = E s_t (the embedding matrix as the output head)."""
    from token_recurrent_decoding_b200 import configs, inputs
    cfg = configs.TINY
    w = {k: v.astype(np.float64) for k, v in inputs.make_weights(cfg, 0, True).items()}
    o = oracle.Oracle(cfg, w)
    s = rng.standard_normal(cfg.d)
    ref = (torch.tensor(w["embed"]) @ torch.tensor(s)).numpy()
    np.testing.assert_allclose(o.lm_head(s), ref, rtol=1e-12, atol=1e-13)


def test_sample_temperature_zero_is_first_argmax():
    lg = np.array([0.5, 2.0, -1.0, 2.0, 1.9])
    assert oracle.sample(lg, 0.0, 0.7) == 1  # the first of the two maxima
    for k in range(20):
        x = rng.standard_normal(33)
        assert oracle.sample(x, 0.0, 0.3) == int(np.argmax(x))


def test_sample_frequencies_on_a_uniform_grid_match_softmax():
    """At u_k = (k + 1/2) / N the draws split into counts N p_v (within one
    per boundary) -- the defining property of inverse-CDF sampling -- with p
    from torch.softmax of logits / temperature."""
    lg = np.array([1.0, -0.5, 0.25, 2.0, -3.0, 0.0, 0.7])
    N = 20000
    for tau in (0.5, 1.0, 2.5):
        counts = np.zeros(lg.size, int)
        for k in range(N):
            counts[oracle.sample(lg, tau, (k + 0.5) / N)] += 1
        p = torch.softmax(torch.tensor(lg) / tau, 0).numpy()
        assert np.all(np.abs(counts - N * p) <= 1.0 + 1e-9), (tau, counts, N * p)


def test_sample_temperature_scales_logits():
    """Temperature tau on logits l draws what temperature 1 draws on l / tau
    (away from CDF boundaries), and the ends of u give the first and the
    last token with weight."""
    lg = rng.standard_normal(50)
    for tau in (0.3, 3.0):
        for u in (0.013, 0.25, 0.5, 0.77, 0.991):
            assert oracle.sample(lg, tau, u) == oracle.sample(lg / tau, 1.0, u)
    assert oracle.sample(lg, 1.0, 0.0) == 0
    assert oracle.sample(lg, 1.0, 1.0 - 1e-15) == lg.size - 1
