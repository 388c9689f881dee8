"""Turn stored inputs (CPU torch tensors) into the oracle's float64 arrays.

TEST INFRASTRUCTURE ONLY (see the package docstring).  bf16 and fp32 values
convert exactly; E4M3 weight codes are decoded with the oracle's own table and
multiplied by their per-output-channel scale; NVFP4 weights likewise.
"""

from __future__ import annotations

import numpy as np
import torch

from .ig4_oracle import dequant_e4m3, dequant_nvfp4


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp16 / fp32 CPU tensor."""
    if t.dtype == torch.float8_e4m3fn:
        raise TypeError("E4M3 codes need their scale: use weight_f64")
    return t.detach().cpu().to(torch.float64).numpy()


def weight_f64(w: torch.Tensor, s: torch.Tensor | None) -> np.ndarray:
    """Linear weight [out, in] as float64 (E4M3 codes decoded and scaled)."""
    if w.dtype == torch.float8_e4m3fn:
        codes = w.detach().cpu().view(torch.uint8).numpy()
        return dequant_e4m3(codes, s.detach().cpu().numpy())
    return to_f64(w)


def block_weights_f64(wt: dict) -> dict:
    """The oracle's weight dict from one block's stored weights (NVFP4 FFN
    weights, recognised by their row-major block scales sfr_*, decoded with
    dequant_nvfp4)."""
    W = {}
    for name in ("w_ada", "w_qkv", "w_o", "w_gate", "w_up", "w_down"):
        sfr = wt.get("sfr" + name[1:])
        if sfr is not None:
            W[name] = dequant_nvfp4(wt[name].cpu().numpy(), sfr.cpu().view(torch.uint8).numpy(),
                                    wt["s" + name[1:]].cpu().numpy())
            continue
        W[name] = weight_f64(wt[name], wt.get("s" + name[1:]))
    W["b_ada"] = to_f64(wt["b_ada"])
    W["g_q"] = to_f64(wt["g_q"])
    W["g_k"] = to_f64(wt["g_k"])
    return W
