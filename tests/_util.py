"""Shared test helpers: error metrics and seeded tensors (no method arithmetic)."""

from __future__ import annotations

import numpy as np
import torch

from synth import tensor_rng


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_abs_over_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / (rms if rms > 0 else 1.0))


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a)))


def randn(name: str, shape, std: float = 1.0, dtype=torch.bfloat16, seed: int = 7) -> torch.Tensor:
    a = tensor_rng(seed, 999, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return torch.from_numpy(a).to(dtype)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


# bf16 unit roundoff: storing a value in bf16 perturbs it by at most this relative amount.
BF16_U = 2.0 ** -8
