"""Helpers for the GPU parity tests: build packed weights through the C-ABI
and measure the error against the fp64 oracle."""
from __future__ import annotations

import numpy as np

TOL = 2e-3   # max relative error, see rel_err


def rel_err(y_gpu_bits: np.ndarray, y_ref: np.ndarray) -> float:
    """max_n |yhat_n - y_n| / max(|y_n|, rms(y)) over each row of [M][N].

    Elementwise relative error is ill-posed where y ~ 0; normalising by
    max(|y_n|, rms(y)) keeps the metric relative for typical outputs and
    absolute (in units of the output RMS) near zero."""
    yg = np.asarray(y_gpu_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    yr = np.atleast_2d(np.asarray(y_ref, dtype=np.float64))
    yg = yg.reshape(yr.shape)
    if not np.array_equal(np.isfinite(yg), np.isfinite(yr)):
        return float("inf")
    worst = 0.0
    for m in range(yr.shape[0]):
        rms = np.sqrt(np.mean(yr[m] ** 2))
        den = np.maximum(np.abs(yr[m]), rms)
        den = np.where(den > 0, den, 1.0)
        worst = max(worst, float(np.max(np.abs(yg[m] - yr[m]) / den)))
    return worst


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def f16_dev(bits: np.ndarray):
    import torch
    return to_dev(np.ascontiguousarray(bits, dtype=np.uint16)).view(torch.float16)


def bits_of(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def packed_on_gpu(eng, gguf: np.ndarray, N: int, K: int):
    g = to_dev(gguf.reshape(-1))
    return eng.repack(g, N, K)
