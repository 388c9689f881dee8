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


__all__ = ["O", "block_weights_f64", "to_f64", "lib", "to_dev", "run_block", "sample_rows",
           "check_output", "rel_l2", "max_abs_over_rms", "rms"]
