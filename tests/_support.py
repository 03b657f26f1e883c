"""Shared test helpers: oracle inputs from generator tensors, parity checks."""
from __future__ import annotations

import numpy as np
import torch

from oracle.inputs import oracle_inputs  # noqa: F401  (re-exported for the GPU tests)


def tolerance(ref_values: np.ndarray) -> float:
    """max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3 (bf16 cache, fp32 accumulate)."""
    return 1e-2 * float(np.max(np.abs(ref_values))) + 1e-3


def compare(gpu_out: torch.Tensor, ref: dict) -> tuple[float, float]:
    """Returns (max abs error, tolerance) over the (b, h) rows in ``ref``."""
    g = gpu_out.double().cpu().numpy()
    keys = sorted(ref)
    R = np.stack([ref[k] for k in keys])
    G = np.stack([g[b, h] for b, h in keys])
    assert np.all(np.isfinite(G)), "non-finite values in the GPU output"
    return float(np.max(np.abs(G - R))), tolerance(R)


def rel_l2(gpu_out: torch.Tensor, ref: dict) -> float:
    g = gpu_out.double().cpu().numpy()
    keys = sorted(ref)
    R = np.stack([ref[k] for k in keys])
    G = np.stack([g[b, h] for b, h in keys])
    return float(np.linalg.norm(G - R) / max(np.linalg.norm(R), 1e-300))
