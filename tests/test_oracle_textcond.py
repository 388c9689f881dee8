"""Pins of the oracle's text conditioning projection (llm_cond_norm +
llm_cond_proj): the feature width the quickstart page prints, closed forms
for constant and one-hot token rows, scale invariance of the norm, token
independence, and a scalar-loop evaluation on a tiny input."""

import numpy as np
import pytest

import oracle as O

RNG = np.random.default_rng(5)


def test_raw_width_is_the_pages_figure():
    # "13 * 4096 = 53,248 float32 values per token"
    assert O.TEXT_RAW_LAYERS * O.TEXT_RAW_WIDTH == 53248


def _problem(M=5, K=96, D=24):
    return (RNG.standard_normal((M, K)), 1.0 + 0.2 * RNG.standard_normal(K),
            RNG.standard_normal((D, K)) / np.sqrt(K), 0.1 * RNG.standard_normal(D))


def test_constant_row_closed_form():
    _, g, w, b = _problem()
    for c in (2.5, -0.75):
        raw = np.full((1, 96), c)
        # RMS of a constant row is |c|: the normed row is c / sqrt(c^2 + eps) * g
        ref = (c / np.sqrt(c * c + 1e-6)) * (w @ g) + b
        assert np.allclose(O.text_cond_projection(raw, g, w, b)[0], ref, rtol=1e-13, atol=1e-13)


def test_one_hot_row_selects_a_weight_column():
    _, g, w, b = _problem()
    K = 96
    raw = np.zeros((1, K))
    raw[0, 17] = 3.0
    # RMS = 3 / sqrt(K): the normed row is sqrt(K) * g[17] (up to eps) at index 17
    scale = 3.0 / np.sqrt(9.0 / K + 1e-6)
    ref = scale * g[17] * w[:, 17] + b
    assert np.allclose(O.text_cond_projection(raw, g, w, b)[0], ref, rtol=1e-12, atol=1e-12)


def test_scale_invariance_and_token_independence():
    raw, g, w, b = _problem()
    out = O.text_cond_projection(raw, g, w, b, eps=0.0)
    assert np.allclose(O.text_cond_projection(7.0 * raw, g, w, b, eps=0.0), out, atol=1e-12)
    perm = np.array([3, 0, 4, 1, 2])
    assert np.allclose(O.text_cond_projection(raw[perm], g, w, b), O.text_cond_projection(raw, g, w, b)[perm],
                       atol=1e-13)
    # batch axes pass through
    out3 = O.text_cond_projection(raw.reshape(1, 5, 96), g, w, b)
    assert out3.shape == (1, 5, 24)


def test_scalar_loops_tiny():
    raw, g, w, b = _problem(M=2, K=8, D=3)
    out = O.text_cond_projection(raw, g, w, b)
    for m in range(2):
        ss = 0.0
        for k in range(8):
            ss += raw[m, k] * raw[m, k]
        r = 1.0 / (ss / 8 + 1e-6) ** 0.5
        for d in range(3):
            acc = b[d]
            for k in range(8):
                acc += raw[m, k] * r * g[k] * w[d, k]
            assert out[m, d] == pytest.approx(acc, rel=1e-12, abs=1e-12)
