"""fp64 CPU oracle of one Ideogram 4 denoising step and of its sampling schedule.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module.  The product path never
imports, links or runs anything under ``oracle/``.

Sources:
  * "Ideogram 4.0" survey page, section "训练方法" (training method): the DiT
    predicts a velocity v(z_t, t) for a flow-matching ODE between pure noise
    and the clean latent; inference integrates it with explicit Euler steps,
    written there as z_{t-dt} = z_t + v * dt; the noise schedule is
    logit-normal (as in SD3), parameterised by (mu, std), with mu shifted by
    resolution as mu_adjusted = mu_base + 0.5 * log(num_pixels / (512 * 512));
    asymmetric classifier-free guidance: the unconditional pass drops the text
    tokens entirely and runs on the image tokens only; the guidance weight
    changes along the trajectory ("polish" tail).
  * the same page, section "Infra", inference engineering: the presets
    V4_QUALITY_48 (48 steps, 45 at gw 7 then 3 at gw 3, mu 0.0, std 1.5),
    V4_DEFAULT_20 (20 steps, 18 at gw 7 then 2 at gw 3, mu 0.0, std 1.75),
    V4_TURBO_12 (12 steps, 11 at gw 7 then 1 at gw 3, mu 0.5, std 1.75).
  * "Ideogram 4 快速开始" (SimpleTuner quickstart), section "验证": the
    unconditional branch is a separate, frozen, image-only transformer, run
    with the text conditioning cleared.

Readings the pages leave open (listed with reasons in the design notes):
  * t runs from 1 (pure noise) down to 0 (clean latent); the N-step schedule
    puts t_i at the (1 - i/N) quantile of the logit-normal distribution
    LN(mu_adjusted, std): t_i = sigmoid(mu_adjusted + std * Phi^-1(1 - i/N)),
    so t_0 = 1 and t_N = 0 exactly;
  * the log in the resolution shift is the natural log;
  * the Euler step is the page's formula with dt = t_i - t_{i+1} > 0:
    z_{i+1} = z_i + (t_i - t_{i+1}) * v, v being the guided velocity;
  * guided velocity v = v_u + gw * (v_c - v_u);
  * the timestep embedding fed to each branch is an input (the pages do not
    describe the timestep embedder).

Every function here is pinned by ``tests/test_oracle_sampler.py``.
"""

from __future__ import annotations

import numpy as np
from scipy.special import expit, ndtri

from .ig4_oracle import mrope_positions, stack_forward

# "Ideogram 4.0" survey page, section "Infra": sampling presets.
GW_MAIN = 7.0
GW_POLISH = 3.0
PRESETS = {
    "V4_QUALITY_48": {"num_steps": 48, "n_polish": 3, "mu": 0.0, "std": 1.5},
    "V4_DEFAULT_20": {"num_steps": 20, "n_polish": 2, "mu": 0.0, "std": 1.75},
    "V4_TURBO_12": {"num_steps": 12, "n_polish": 1, "mu": 0.5, "std": 1.75},
}


def resolution_mu(mu_base: float, height: int, width: int) -> float:
    """mu_adjusted = mu_base + 0.5 * ln(height * width / 512^2)."""
    return float(mu_base) + 0.5 * np.log(float(height) * float(width) / (512.0 * 512.0))


def flow_schedule(num_steps: int, mu_base: float, std: float, height: int, width: int) -> np.ndarray:
    """Times t_0 = 1 > t_1 > ... > t_N = 0 of an N-step sampler (float64, N + 1).

    t_i is the (1 - i/N) quantile of the logit-normal distribution with
    location mu_adjusted (the resolution-shifted mu) and scale std.
    """
    n = int(num_steps)
    mu = resolution_mu(mu_base, height, width)
    p = 1.0 - np.arange(n + 1, dtype=np.float64) / n
    return expit(mu + float(std) * ndtri(p))


def guidance_schedule(num_steps: int, n_polish: int, gw_main: float = GW_MAIN,
                      gw_polish: float = GW_POLISH) -> np.ndarray:
    """Guidance weight of each of the N steps: gw_main, then gw_polish for the
    last n_polish steps (the "polish" tail near t = 0)."""
    gw = np.full(int(num_steps), float(gw_main), dtype=np.float64)
    if n_polish > 0:
        gw[num_steps - n_polish:] = float(gw_polish)
    return gw


def cfg_velocity(v_cond: np.ndarray, v_uncond: np.ndarray, gw: float) -> np.ndarray:
    """Classifier-free guidance: v = v_u + gw * (v_c - v_u)."""
    v_cond = np.asarray(v_cond, dtype=np.float64)
    v_uncond = np.asarray(v_uncond, dtype=np.float64)
    return v_uncond + float(gw) * (v_cond - v_uncond)


def euler_update(z: np.ndarray, v: np.ndarray, t_cur: float, t_next: float) -> np.ndarray:
    """One explicit Euler step from t_cur down to t_next: z + (t_cur - t_next) * v."""
    return np.asarray(z, dtype=np.float64) + (float(t_cur) - float(t_next)) * np.asarray(v, dtype=np.float64)


def denoise_step(z, text, temb_cond, temb_uncond, t_cur, t_next, gw, grid, cond, uncond, H, **kw):
    """One full sampler step with asymmetric CFG, float64.

    z: latent [B, N, C]; text: [B, T, D] (the conditional branch's prefix);
    grid: (grid_t, grid_h, grid_w) with N = grid_t * grid_h * grid_w; cond and
    uncond: dicts with the stack weights (keys block_weights, n_blocks, w_in,
    b_in, w_f, b_f, w_out, b_out) of the conditional transformer and of the
    separate image-only unconditional transformer.  The conditional pass runs
    on [text | image]; the unconditional one on the image tokens alone, with
    image positions computed for an empty text prefix.
    """
    text = np.asarray(text, dtype=np.float64)
    B, T = text.shape[0], text.shape[1]
    gt, gh, gwid = grid
    pos_c = mrope_positions(T, gt, gh, gwid)
    pos_u = mrope_positions(0, gt, gh, gwid)
    v_c = stack_forward(z, text, temb_cond, pos_c, cond["block_weights"], cond["n_blocks"],
                        cond["w_in"], cond["b_in"], cond["w_f"], cond["b_f"], cond["w_out"],
                        cond["b_out"], H, **kw)
    no_text = np.zeros((B, 0, text.shape[2]), dtype=np.float64)
    v_u = stack_forward(z, no_text, temb_uncond, pos_u, uncond["block_weights"], uncond["n_blocks"],
                        uncond["w_in"], uncond["b_in"], uncond["w_f"], uncond["b_f"],
                        uncond["w_out"], uncond["b_out"], H, **kw)
    return euler_update(z, cfg_velocity(v_c, v_u, gw), t_cur, t_next)
