"""Helpers shared by the GPU parity tests: device copies of the seeded inputs,
the library handle, sampled rows, and the acceptance metrics."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
from oracle.inputs import block_weights_f64, to_f64
from tests._util import BF16_U, max_abs_over_rms, rel_l2, rms


def lib():
    from stream_diffusion_transformer_fwd_b200.build import build
    build()
    from stream_diffusion_transformer_fwd_b200 import ig4
    return ig4


def to_dev(d: dict, device="cuda") -> dict:
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def run_block(ig4, cfg, w_dev, x, temb, pos=None, out=None):
    """ig4_block_forward on device tensors; returns x_out."""
    c = ig4.config_from(cfg)
    if pos is None:
        pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w,
                                      device=x.device)
    ws = torch.empty(ig4.ig4_workspace_size(c), dtype=torch.uint8, device=x.device)
    out = torch.empty_like(x) if out is None else out
    ig4.ig4_block_forward(c, ig4.block_weights(w_dev), x, out, pos, temb, ws)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return out


def sample_rows(cfg, n=48, seed=3) -> np.ndarray:
    """Token rows to check at full size: both ends, the text/image boundary,
    tile boundaries, the ragged tail, and a seeded random spread."""
    L, M = cfg.L, cfg.M
    fixed = [0, 1, 127, 128, cfg.T_text - 1, cfg.T_text, L - 1, M - 1, M // 2]
    rng = np.random.default_rng(seed)
    rnd = rng.choice(M, size=n, replace=False)
    return np.unique(np.clip(np.array(fixed + list(rnd)), 0, M - 1))


def delta_tolerance(base_tol: float, y_ref: np.ndarray, d_ref: np.ndarray, stored_bf16: bool):
    """Tolerance on delta = y - x.  When the residual stream is stored in bf16,
    x1 and y each take one bf16 rounding (relative error <= 2^-8) that is of
    the size of the stream, not of delta; scale that by RMS(y)/RMS(delta)."""
    if not stored_bf16:
        return base_tol
    return base_tol + 2.0 * BF16_U * rms(y_ref) / max(rms(d_ref), 1e-30)


def check_output(y_gpu: np.ndarray, y_ref: np.ndarray, x: np.ndarray, fp8: bool,
                 stored_bf16: bool, what=""):
    """Acceptance: y within rel-L2 1e-2 and max-abs 5e-2 RMS (bf16) or rel-L2
    3e-2 (FP8 weights); delta = y - x within the derived tolerance."""
    tol = 3e-2 if fp8 else 1e-2
    e_y = rel_l2(y_gpu, y_ref)
    m_y = max_abs_over_rms(y_gpu, y_ref)
    d_ref = y_ref - x
    d_gpu = y_gpu - x
    e_d = rel_l2(d_gpu, d_ref)
    tol_d = delta_tolerance(2.0 * tol, y_ref, d_ref, stored_bf16)
    msg = f"{what}: relL2(y)={e_y:.3e} maxabs/rms(y)={m_y:.3e} relL2(delta)={e_d:.3e} (tol {tol_d:.3e})"
    print(msg)
    assert e_y <= tol, msg
    if not fp8:
        assert m_y <= 5e-2, msg
    assert e_d <= tol_d, msg
    return e_y, m_y, e_d


def live_blocks(cfg, host_blocks: dict, seed: int) -> list:
    """Device weights of cfg.n_blocks blocks: block i takes the host-drawn
    weights host_blocks[i] where given, else weights drawn on the device
    (synth.make_block_weights_device: same shapes and distributions, their
    values never reach the oracle)."""
    from synth import make_block_weights_device

    return [to_dev(host_blocks[i]) if i in host_blocks
            else make_block_weights_device(cfg, seed, i, "cuda") for i in range(cfg.n_blocks)]


def stack_weights_dev(ig4, cfg, st, blocks):
    """(StackWeights, device copies of the stack-level inputs) for a stack call."""
    sd = to_dev(st)
    sw = ig4.stack_weights([ig4.block_weights(b) for b in blocks], sd["w_in"], sd["s_in"],
                           sd["b_in"], sd["w_f"], sd["s_f"], sd["b_f"], sd["w_out"], sd["s_out"],
                           sd["b_out"], cfg.latent_ch)
    return sw, sd


def run_stack_tapped(ig4, cfg, st, blocks, tap_ids, x_latent):
    """ig4_stack_forward_tapped over the device blocks `blocks`, tapping the
    sequence entering each block in tap_ids (cfg.n_blocks: after the last).
    Returns (out_latent device tensor, {block index: sequence as float64})."""
    c = ig4.config_from(cfg)
    sw, sd = stack_weights_dev(ig4, cfg, st, blocks)
    pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w, device="cuda")
    ws = torch.empty(ig4.ig4_stack_workspace_size(c, cfg.latent_ch), dtype=torch.uint8,
                     device="cuda")
    taps = {i: torch.empty(cfg.B, cfg.L, cfg.D, dtype=torch.bfloat16, device="cuda")
            for i in sorted(tap_ids)}
    lat = x_latent.cuda()
    out = torch.empty_like(lat)
    ig4.ig4_stack_forward_tapped(c, sw, lat, sd["text"] if cfg.T_text > 0 else None, out, pos,
                                 sd["temb"], ws, taps)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return out, {i: t.float().cpu().double().numpy() for i, t in taps.items()}


def tap_ids_for(cfg, host_blocks: dict) -> set:
    """Taps check_tapped_stack needs: into and out of each checked block, and
    the sequence after the last block."""
    return {j for i in host_blocks for j in (i, i + 1)} | {0, cfg.n_blocks}


def check_tapped_stack(cfg, st, host_blocks: dict, seq: dict, out, x_latent64, n_rows=48):
    """A tapped stack against the oracle: the sequence entering block 0 against
    stack_input of the stack's inputs (every element, bf16 tolerance); each
    host block on sampled token rows (the oracle's block_forward_rows of the
    tapped input, FP8 or bf16 tolerance by cfg.w_dtype); the final layer of
    the tapped last sequence against out_latent (every element)."""
    from oracle.inputs import weight_f64

    fp8 = cfg.w_dtype == "e4m3"
    temb = to_f64(st["temb"])
    text = to_f64(st["text"]) if cfg.T_text > 0 else np.zeros((cfg.B, 0, cfg.D))
    s0 = O.stack_input(x_latent64, text, weight_f64(st["w_in"], st["s_in"]), to_f64(st["b_in"]))
    e0, m0 = rel_l2(seq[0], s0), max_abs_over_rms(seq[0], s0)
    print(f"{cfg.name} stack input: relL2={e0:.3e} maxabs/rms={m0:.3e}")
    assert e0 <= 1e-2 and m0 <= 5e-2
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    rows = sample_rows(cfg, n=n_rows)
    for i in sorted(host_blocks):
        x_i = seq[i]
        y_ref = O.block_forward_rows(x_i, temb, pos, block_weights_f64(host_blocks[i]), cfg.H,
                                     rows, cfg.rope_theta, cfg.sections, cfg.eps)
        y_i = seq[i + 1].reshape(cfg.M, cfg.D)[rows]
        check_output(y_i, y_ref, x_i.reshape(cfg.M, cfg.D)[rows], fp8, True,
                     f"{cfg.name} block {i}")
    ref = O.final_layer(seq[cfg.n_blocks], temb, cfg.T_text, weight_f64(st["w_f"], st["s_f"]),
                        to_f64(st["b_f"]), weight_f64(st["w_out"], st["s_out"]),
                        to_f64(st["b_out"]), cfg.eps)
    out = out.float().cpu().double().numpy() if isinstance(out, torch.Tensor) else out
    e, m = rel_l2(out, ref), max_abs_over_rms(out, ref)
    print(f"{cfg.name} final layer: relL2={e:.3e} maxabs/rms={m:.3e}")
    assert e <= 1e-2 and m <= 5e-2


__all__ = ["O", "block_weights_f64", "to_f64", "lib", "to_dev", "run_block", "sample_rows",
           "check_output", "live_blocks", "stack_weights_dev", "run_stack_tapped",
           "tap_ids_for", "check_tapped_stack", "rel_l2",
           "max_abs_over_rms", "rms"]
