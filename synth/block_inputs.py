"""Seeded draws of the block's weights and activations.

Distributions (the workload description): activations, text tokens, latents
and the timestep embedding ~ N(0, 1); linear weights ~ N(0, 1/fan_in); the
AdaLN projections ~ N(0, 0.02^2); biases 0; QK-norm weights 1.  ``stress=True``
draws non-trivial biases (N(0, 0.1^2)) and QK-norm weights (1 + N(0, 0.2^2))
so that a dropped bias or norm weight shows up in parity.

FP8 weights use the release format: E4M3 ("fn", max 448) codes with a
per-output-channel fp32 scale s[n] = max_k |W[n, k]| / 448, codes rounded to
nearest even from W / s.  Everything is returned as CPU torch tensors.
"""

from __future__ import annotations

import zlib

import numpy as np
import torch

from .configs import Config

E4M3_MAX = 448.0


def tensor_rng(seed: int, block: int, name: str) -> np.random.Generator:
    """One independent numpy stream per (seed, block, tensor name)."""
    return np.random.default_rng([int(seed), int(block), zlib.crc32(name.encode())])


def _normal(seed, block, name, shape, std=1.0) -> np.ndarray:
    a = tensor_rng(seed, block, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def quantize_e4m3_per_channel(w: np.ndarray):
    """fp32 [N, K] -> (E4M3 codes as torch.float8_e4m3fn [N, K], fp32 scale [N])."""
    w = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32))
    amax = w.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (w / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q, scale.to(torch.float32)


def _linear(seed, block, name, n_out, n_in, w_dtype, std=None):
    """Weight [n_out, n_in] (+ scale for E4M3, else None)."""
    std = (1.0 / np.sqrt(n_in)) if std is None else std
    w = _normal(seed, block, name, (n_out, n_in), std)
    if w_dtype == "bf16":
        return torch.from_numpy(w).to(torch.bfloat16), None
    if w_dtype == "e4m3":
        return quantize_e4m3_per_channel(w)
    raise ValueError(f"w_dtype {w_dtype!r}")


def _bias(seed, block, name, n, stress):
    if stress:
        return torch.from_numpy(_normal(seed, block, name, (n,), 0.1))
    return torch.zeros(n, dtype=torch.float32)


def make_block_weights(cfg: Config, seed: int = 0, block: int = 0, stress: bool = False,
                       zero_adaln: bool = False) -> dict:
    """Weights of one block: w_* [out, in] (bf16 or E4M3 codes), s_* fp32 scales
    (E4M3 only, else None), b_ada fp32 [6D], g_q / g_k fp32 [head_dim].  With
    w_dtype "nvfp4_mixed" the FFN weights are NVFP4 (see make_nvfp4_linear:
    w_* codes, sfr_* row-major block scales, s_* channel scales)."""
    D, I, A, dh = cfg.D, cfg.I, cfg.adaln_dim, cfg.head_dim
    wd = cfg.w_dtype
    wa = "e4m3" if wd == "nvfp4_mixed" else wd  # AdaLN and attention projections
    out = {}
    out["w_ada"], out["s_ada"] = _linear(seed, block, "w_ada", 6 * D, A, wa, std=0.02)
    if zero_adaln:
        out["w_ada"] = torch.zeros_like(out["w_ada"])
    out["b_ada"] = torch.zeros(6 * D) if zero_adaln else _bias(seed, block, "b_ada", 6 * D, stress)
    out["w_qkv"], out["s_qkv"] = _linear(seed, block, "w_qkv", 3 * D, D, wa)
    out["w_o"], out["s_o"] = _linear(seed, block, "w_o", D, D, wa)
    if wd == "nvfp4_mixed":
        # FFN linears in NVFP4 (E2M1 codes, row-major E4M3 block scales sfr_*,
        # channel scales s_*); every other linear in E4M3
        for name, n_out, n_in in (("gate", I, D), ("up", I, D), ("down", D, I)):
            q = make_nvfp4_linear(seed, block, "w_" + name, n_out, n_in)
            out["w_" + name], out["sfr_" + name], out["s_" + name] = q["codes"], q["sf"], q["s"]
    else:
        out["w_gate"], out["s_gate"] = _linear(seed, block, "w_gate", I, D, wd)
        out["w_up"], out["s_up"] = _linear(seed, block, "w_up", I, D, wd)
        out["w_down"], out["s_down"] = _linear(seed, block, "w_down", D, I, wd)
    if stress:
        out["g_q"] = torch.from_numpy(1.0 + _normal(seed, block, "g_q", (dh,), 0.2))
        out["g_k"] = torch.from_numpy(1.0 + _normal(seed, block, "g_k", (dh,), 0.2))
    else:
        out["g_q"] = torch.ones(dh, dtype=torch.float32)
        out["g_k"] = torch.ones(dh, dtype=torch.float32)
    return out


def make_block_activations(cfg: Config, seed: int = 0) -> dict:
    """x [B, L, D] (fp32 or bf16 per cfg.x_dtype) and temb [B, adaln_dim] fp32."""
    x = torch.from_numpy(_normal(seed, 0, "x", (cfg.B, cfg.L, cfg.D)))
    if cfg.x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    elif cfg.x_dtype != "f32":
        raise ValueError(f"x_dtype {cfg.x_dtype!r}")
    temb = torch.from_numpy(_normal(seed, 0, "temb", (cfg.B, cfg.adaln_dim)))
    return {"x": x, "temb": temb}


def make_block_weights_device(cfg: Config, seed: int, block: int, device) -> dict:
    """Weights of one block drawn on `device` with a seeded torch generator.

    Same shapes, distributions and storage formats as make_block_weights
    (E4M3 codes with per-output-channel scales for FP8), but not the same
    values: meant for timing full-size stacks, whose 9.3e9 parameters would
    take minutes to draw on the host.  Parity tests use make_block_weights.
    """
    D, I, A, dh = cfg.D, cfg.I, cfg.adaln_dim, cfg.head_dim
    gen = torch.Generator(device=device)

    def draw(name, n_out, n_in, std):
        gen.manual_seed(zlib.crc32(f"{seed}/{block}/{name}".encode()))
        w = torch.randn((n_out, n_in), generator=gen, device=device, dtype=torch.float32) * std
        if cfg.w_dtype == "bf16":
            return w.to(torch.bfloat16), None
        amax = w.abs().amax(dim=1)
        scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        q = (w / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
        return q, scale

    out = {}
    out["w_ada"], out["s_ada"] = draw("w_ada", 6 * D, A, 0.02)
    out["b_ada"] = torch.zeros(6 * D, device=device)
    out["w_qkv"], out["s_qkv"] = draw("w_qkv", 3 * D, D, 1.0 / np.sqrt(D))
    out["w_o"], out["s_o"] = draw("w_o", D, D, 1.0 / np.sqrt(D))
    out["w_gate"], out["s_gate"] = draw("w_gate", I, D, 1.0 / np.sqrt(D))
    out["w_up"], out["s_up"] = draw("w_up", I, D, 1.0 / np.sqrt(D))
    out["w_down"], out["s_down"] = draw("w_down", D, I, 1.0 / np.sqrt(I))
    out["g_q"] = torch.ones(dh, device=device)
    out["g_k"] = torch.ones(dh, device=device)
    return out


def make_stack_inputs(cfg: Config, seed: int = 0, stress: bool = False) -> dict:
    """Stack-level inputs: latents [B, N, C] and text [B, T, D] (x_dtype), temb fp32,
    in-proj w_in [D, C] / b_in, final AdaLN w_f [2D, A] / b_f, out-proj w_out [C, D] /
    b_out (weights in cfg.w_dtype with scales for E4M3).  Block weights come from
    make_block_weights(cfg, seed, block=i)."""
    D, A, C = cfg.D, cfg.adaln_dim, cfg.latent_ch
    xd = torch.bfloat16 if cfg.x_dtype == "bf16" else torch.float32
    wd = "e4m3" if cfg.w_dtype == "nvfp4_mixed" else cfg.w_dtype  # only the FFN is NVFP4
    out = {}
    out["x_latent"] = torch.from_numpy(_normal(seed, 0, "x_latent", (cfg.B, cfg.n_img, C))).to(xd)
    out["text"] = torch.from_numpy(_normal(seed, 0, "text", (cfg.B, cfg.T_text, D))).to(xd)
    out["temb"] = torch.from_numpy(_normal(seed, 0, "temb", (cfg.B, A)))
    out["w_in"], out["s_in"] = _linear(seed, 0, "w_in", D, C, wd)
    out["b_in"] = _bias(seed, 0, "b_in", D, stress)
    out["w_f"], out["s_f"] = _linear(seed, 0, "w_f", 2 * D, A, wd, std=0.02)
    out["b_f"] = _bias(seed, 0, "b_f", 2 * D, stress)
    out["w_out"], out["s_out"] = _linear(seed, 0, "w_out", C, D, wd)
    out["b_out"] = _bias(seed, 0, "b_out", C, stress)
    return out


def make_text_cond_inputs(M: int, K_raw: int, D: int, w_dtype: str = "bf16", seed: int = 0,
                          stress: bool = False) -> dict:
    """Inputs of the text conditioning projection: raw fp32 [M, K_raw] ~ N(0, 1)
    (concatenated text-encoder features), g_norm fp32 [K_raw] (1, or 1 + N(0, 0.2^2)
    with stress), w_proj [D, K_raw] ~ N(0, 1/K_raw) (+ scale for E4M3), b_proj
    fp32 [D] (0, or N(0, 0.1^2) with stress)."""
    out = {"raw": torch.from_numpy(_normal(seed, 0, "text_raw", (M, K_raw)))}
    if stress:
        out["g_norm"] = torch.from_numpy(1.0 + _normal(seed, 0, "g_text", (K_raw,), 0.2))
    else:
        out["g_norm"] = torch.ones(K_raw, dtype=torch.float32)
    out["w_proj"], out["s_proj"] = _linear(seed, 0, "w_text_proj", D, K_raw, w_dtype)
    out["b_proj"] = _bias(seed, 0, "b_text_proj", D, stress)
    return out


# ----------------------------------------------------------------- NVFP4
# E2M1 ("fp4"): sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes of
# codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


_E2M1_MID = 0.5 * (_E2M1_MAG[1:] + _E2M1_MAG[:-1])  # decision points between codes


def _e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code of each value (ties to the even code), saturating at
    +-6; returns uint8 codes 0..15 (bit 3 = sign)."""
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    idx = np.searchsorted(_E2M1_MID, a, side="left")  # midpoints strictly below a
    tie = (idx < 7) & (a == _E2M1_MID[np.minimum(idx, 6)])
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx).astype(np.uint8)
    sign = ((v < 0) & (idx > 0)).astype(np.uint8) << 3
    return idx | sign


def _e4m3_round(v: np.ndarray) -> torch.Tensor:
    """fp32 -> E4M3 (round to nearest even, saturating to +-448)."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return t.clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)


def quantize_nvfp4(w: np.ndarray, block: int = 64):
    """fp32 [N, K] -> (codes uint8 [N, K/2], element 2i in the low nibble;
    block scales E4M3 [N, K/16], each `block`-element block's scale repeated
    over its 16-element sub-blocks; per-row fp32 scale [N]).

    W[n, k] ~= s[n] * sb[n, k // 16] * e2m1(code[n, k]); s[n] = max|W[n]| /
    (6 * 448) puts the largest block scale at 448, sb = RNE_E4M3(block amax /
    (6 s[n])), codes = RNE_E2M1(W / (s sb))."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % block == 0 and block % 16 == 0
    amax = np.abs(w).max(axis=1)
    s = np.where(amax > 0, amax / (6.0 * E4M3_MAX), 1.0).astype(np.float32)
    bam = np.abs(w.reshape(N, K // block, block)).max(axis=2)
    sb = _e4m3_round(bam / (6.0 * s[:, None]))
    sbf = sb.to(torch.float32).numpy().astype(np.float64)
    denom = np.repeat(s[:, None].astype(np.float64) * sbf, block, axis=1)
    q = np.where(denom > 0, w / np.where(denom > 0, denom, 1.0), 0.0)
    codes = _e2m1_encode(q)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    sb16 = np.repeat(sb.view(torch.uint8).numpy(), block // 16, axis=1)
    return (torch.from_numpy(packed), torch.from_numpy(np.ascontiguousarray(sb16)).view(torch.float8_e4m3fn),
            torch.from_numpy(s))


def make_nvfp4_linear(seed: int, block: int, name: str, n_out: int, n_in: int, std=None,
                      block_elems: int = 64) -> dict:
    """A linear layer's weight [n_out, n_in] ~ N(0, 1/n_in) in NVFP4 (see
    quantize_nvfp4); keys codes, sf (E4M3 [n_out, n_in/16]), s (fp32 [n_out])."""
    std = (1.0 / np.sqrt(n_in)) if std is None else std
    w = _normal(seed, block, name, (n_out, n_in), std)
    codes, sf, s = quantize_nvfp4(w, block_elems)
    return {"codes": codes, "sf": sf, "s": s}
