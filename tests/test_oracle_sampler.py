"""Pins of the sampler oracle (schedule, guidance, Euler step, denoising step).

Closed forms of the logit-normal quantile schedule, the inverse check of every
time against an independent normal CDF (math.erfc), the presets as the survey
page prints them, exact integration of straight-line flows by the Euler step,
and invariants of asymmetric classifier-free guidance.
"""

import math
import os

import numpy as np
import pytest

import oracle as O
from oracle import ig4_sampler as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sampler_presets.txt")
RNG = np.random.default_rng(91)


def _presets():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, n, n_main, gw_main, n_pol, gw_pol, mu, std = line.split()
            rows.append((name, int(n), int(n_main), float(gw_main), int(n_pol), float(gw_pol),
                         float(mu), float(std)))
    return rows


def _phi(x):
    """Standard normal CDF from math.erfc (independent of scipy's ndtri)."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def test_presets_match_the_page():
    rows = _presets()
    assert len(rows) == 3
    for name, n, n_main, gw_main, n_pol, gw_pol, mu, std in rows:
        p = S.PRESETS[name]
        assert (p["num_steps"], p["n_polish"], p["mu"], p["std"]) == (n, n_pol, mu, std)
        assert n_main + n_pol == n
        gw = S.guidance_schedule(p["num_steps"], p["n_polish"])
        assert list(gw) == [gw_main] * n_main + [gw_pol] * n_pol


def test_resolution_shift_closed_forms():
    assert S.resolution_mu(0.3, 512, 512) == 0.3
    assert S.resolution_mu(0.0, 1024, 1024) == pytest.approx(math.log(2.0), abs=1e-15)
    assert S.resolution_mu(0.5, 256, 256) == pytest.approx(0.5 - math.log(2.0), abs=1e-15)
    assert S.resolution_mu(0.0, 2048, 352) == pytest.approx(0.5 * math.log(2048 * 352 / 512 ** 2),
                                                            abs=1e-15)


@pytest.mark.parametrize("n,mu,std,h,w", [(48, 0.0, 1.5, 1024, 1024), (20, 0.0, 1.75, 512, 512),
                                          (12, 0.5, 1.75, 2048, 352), (7, -0.3, 0.8, 256, 1536)])
def test_schedule_endpoints_monotone_and_quantiles(n, mu, std, h, w):
    t = S.flow_schedule(n, mu, std, h, w)
    assert t.shape == (n + 1,)
    assert t[0] == 1.0 and t[-1] == 0.0
    assert np.all(np.diff(t) < 0)
    mu_adj = S.resolution_mu(mu, h, w)
    for i in range(1, n):
        # t_i is the (1 - i/N) quantile of LN(mu_adj, std): invert it with the CDF
        z = (math.log(t[i] / (1.0 - t[i])) - mu_adj) / std
        assert _phi(z) == pytest.approx(1.0 - i / n, abs=1e-12)


def test_schedule_middle_step_closed_form():
    # N even: the middle quantile is the median, sigmoid(mu_adj); at 1024 x 1024
    # and mu = 0 that is sigmoid(ln 2) = 2/3.
    t = S.flow_schedule(48, 0.0, 1.5, 1024, 1024)
    assert t[24] == pytest.approx(2.0 / 3.0, abs=1e-15)
    t = S.flow_schedule(20, 0.5, 1.75, 512, 512)
    assert t[10] == pytest.approx(1.0 / (1.0 + math.exp(-0.5)), abs=1e-15)
    # a vanishing std collapses every interior step onto the median
    t = S.flow_schedule(9, 0.2, 1e-12, 512, 512)
    assert np.allclose(t[1:-1], 1.0 / (1.0 + math.exp(-0.2)), atol=1e-10)


def test_schedule_larger_mu_spends_more_steps_at_high_noise():
    lo = S.flow_schedule(20, 0.0, 1.75, 512, 512)
    hi = S.flow_schedule(20, 0.0, 1.75, 2048, 2048)
    assert np.all(hi[1:-1] > lo[1:-1])


def test_guidance_schedule_edges():
    assert list(S.guidance_schedule(4, 0, 5.0, 1.0)) == [5.0] * 4
    assert list(S.guidance_schedule(4, 4, 5.0, 1.0)) == [1.0] * 4


def test_cfg_velocity_weights():
    vc, vu = RNG.standard_normal((2, 5, 8)), RNG.standard_normal((2, 5, 8))
    assert np.array_equal(S.cfg_velocity(vc, vu, 1.0), vu + (vc - vu))
    assert np.allclose(S.cfg_velocity(vc, vu, 1.0), vc, atol=1e-15)
    assert np.array_equal(S.cfg_velocity(vc, vu, 0.0), vu)
    # linear in the weight
    a, b = S.cfg_velocity(vc, vu, 2.0), S.cfg_velocity(vc, vu, 5.0)
    assert np.allclose(S.cfg_velocity(vc, vu, 3.5), 0.5 * (a + b), atol=1e-13)


def test_euler_integrates_straight_flows_exactly():
    # Straight path from noise e (t = 1) to data x0 (t = 0): z_t = (1 - t) x0 + t e.
    # Its velocity toward the data, x0 - e, is constant, so Euler steps with the
    # page's update z_{t-dt} = z_t + v dt reach x0 on any schedule.
    x0, e = RNG.standard_normal((3, 16)), RNG.standard_normal((3, 16))
    for n, mu, std in [(48, 0.0, 1.5), (12, 0.5, 1.75), (3, 1.0, 0.5)]:
        t = S.flow_schedule(n, mu, std, 1024, 1024)
        z = e.copy()
        for i in range(n):
            z = S.euler_update(z, x0 - e, t[i], t[i + 1])
            assert np.allclose(z, (1 - t[i + 1]) * x0 + t[i + 1] * e, atol=1e-12)
        assert np.allclose(z, x0, atol=1e-12)


def _tiny_stack(D, H, I, A, C, seed, zero_gates=False):
    rng = np.random.default_rng(seed)
    dh = D // H

    def block(i):
        r = np.random.default_rng([seed, i])
        w = {
            "w_ada": r.standard_normal((6 * D, A)) * 0.02,
            "b_ada": r.standard_normal(6 * D) * 0.1,
            "w_qkv": r.standard_normal((3 * D, D)) / np.sqrt(D),
            "g_q": np.ones(dh), "g_k": np.ones(dh),
            "w_o": r.standard_normal((D, D)) / np.sqrt(D),
            "w_gate": r.standard_normal((I, D)) / np.sqrt(D),
            "w_up": r.standard_normal((I, D)) / np.sqrt(D),
            "w_down": r.standard_normal((D, I)) / np.sqrt(I),
        }
        if zero_gates:
            w["w_ada"][:] = 0.0
            w["b_ada"][:] = 0.0
        return w

    return {"block_weights": block, "n_blocks": 2,
            "w_in": rng.standard_normal((D, C)) / np.sqrt(C), "b_in": rng.standard_normal(D) * 0.1,
            "w_f": rng.standard_normal((2 * D, A)) * 0.02, "b_f": rng.standard_normal(2 * D) * 0.1,
            "w_out": rng.standard_normal((C, D)) / np.sqrt(D), "b_out": rng.standard_normal(C) * 0.1}


def _step_inputs(B=1, T=3, grid=(1, 2, 3), D=512, A=16, C=16):
    N = grid[0] * grid[1] * grid[2]
    return (RNG.standard_normal((B, N, C)), RNG.standard_normal((B, T, D)),
            RNG.standard_normal((B, A)), RNG.standard_normal((B, A)))


def test_denoise_step_guidance_invariants():
    D, H, I, A, C = 512, 2, 64, 16, 16
    grid = (1, 2, 3)
    z, text, tc, tu = _step_inputs(grid=grid)
    cond, uncond = _tiny_stack(D, H, I, A, C, 1), _tiny_stack(D, H, I, A, C, 2)
    # gw = 1: the step follows the conditional velocity and ignores the
    # unconditional transformer entirely
    a = S.denoise_step(z, text, tc, tu, 0.8, 0.6, 1.0, grid, cond, uncond, H)
    other = _tiny_stack(D, H, I, A, C, 3)
    b = S.denoise_step(z, text, tc, tu, 0.8, 0.6, 1.0, grid, cond, other, H)
    assert np.allclose(a, b, rtol=0, atol=1e-12)
    # gw = 0: the step follows the unconditional velocity, which never sees the text
    c0 = S.denoise_step(z, text, tc, tu, 0.8, 0.6, 0.0, grid, cond, uncond, H)
    c1 = S.denoise_step(z, 5.0 * text, tc, tu, 0.8, 0.6, 0.0, grid, cond, uncond, H)
    assert np.array_equal(c0, c1)
    assert not np.allclose(a, c0)
    # the unconditional branch is the stack over the image tokens alone, with
    # the image positions of an empty text prefix
    v_u = (c0 - z) / 0.2
    ref = O.stack_forward(z, np.zeros((1, 0, D)), tu, O.mrope_positions(0, *grid),
                          uncond["block_weights"], 2, uncond["w_in"], uncond["b_in"], uncond["w_f"],
                          uncond["b_f"], uncond["w_out"], uncond["b_out"], H)
    assert np.allclose(v_u, ref, atol=1e-10)
    # same transformer and no text on either side: the guidance weight drops out
    z2, _, t2, _ = _step_inputs(T=0, grid=grid)
    empty = np.zeros((1, 0, D))
    d1 = S.denoise_step(z2, empty, t2, t2, 0.5, 0.25, 7.0, grid, cond, cond, H)
    d2 = S.denoise_step(z2, empty, t2, t2, 0.5, 0.25, 3.0, grid, cond, cond, H)
    assert np.allclose(d1, d2, atol=1e-12)


def test_denoise_step_zero_gates_closed_form():
    # Zero block gates make both stacks in-proj -> final norm -> out-proj, so the
    # whole step is a closed form of the latent.
    D, H, I, A, C = 512, 2, 64, 16, 16
    grid = (1, 2, 2)
    z, text, tc, tu = _step_inputs(grid=grid, T=2)
    cond, uncond = _tiny_stack(D, H, I, A, C, 4, True), _tiny_stack(D, H, I, A, C, 5, True)

    def head(p, temb):
        img = z @ p["w_in"].T + p["b_in"]
        c = temb / (1 + np.exp(-temb))
        mod = c @ p["w_f"].T + p["b_f"]
        sh, sc = mod[:, :D], mod[:, D:]
        r = 1.0 / np.sqrt(np.mean(img ** 2, axis=-1, keepdims=True) + 1e-6)
        return (img * r * (1 + sc[:, None]) + sh[:, None]) @ p["w_out"].T + p["b_out"]

    vc, vu = head(cond, tc), head(uncond, tu)
    got = S.denoise_step(z, text, tc, tu, 0.9, 0.7, 4.0, grid, cond, uncond, H)
    assert np.allclose(got, z + 0.2 * (vu + 4.0 * (vc - vu)), rtol=1e-12, atol=1e-12)
