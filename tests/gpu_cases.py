"""Shared helpers for the GPU parity tests: seeded inputs drawn on the CPU
(the same bytes go to the oracle and to the device) and the comparison
metrics the parity bar is stated in."""
from __future__ import annotations

import numpy as np
import torch

from bitlinear_rmsnorm_quant_b200 import inputs as I

# End-to-end bar on y: max relative error 1e-2, relative to max(|y_ref|,
# 1e-2 * rms of the token's y_ref row) so that outputs near zero do not
# dominate; at most 0.1% of int8 activation codes may differ, and only by one.
Y_REL_TOL = 1e-2
Y_FLOOR = 1e-2
Q_MAX_DIFF_FRAC = 1e-3


def bits_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def make_layer(seed: int, M: int, K: int, N: int, index: int = 0, outlier_frac: float = 0.0):
    """CPU tensors x (bf16), gamma (fp32), W (fp32) of one projection."""
    x = I.activations(seed, M, K, index=index, outlier_frac=outlier_frac)
    g = I.gamma(seed, K, index=index)
    W = I.latent_weights(seed, N, K, index=index)
    return x, g, W


def y_rel_error(y: np.ndarray, y_ref: np.ndarray) -> float:
    """max |y - y_ref| / max(|y_ref|, 1e-2 * rms(y_ref row)) over all elements."""
    yv = bf16_to_f64(y)
    rv = bf16_to_f64(y_ref)
    if rv.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(rv * rv, axis=1, keepdims=True))
    den = np.maximum(np.abs(rv), Y_FLOOR * rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(yv - rv) / den))


def q_diff_stats(q: np.ndarray, q_ref: np.ndarray):
    d = np.abs(q.astype(np.int32) - q_ref.astype(np.int32))
    return float((d != 0).mean()) if d.size else 0.0, int(d.max()) if d.size else 0
