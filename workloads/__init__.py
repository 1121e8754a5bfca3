"""Seeded synthetic inputs for the fake-quant workloads.

This module is the only code shared by the oracle side and the CUDA side: it
draws random numbers and rounds them to BF16 with torch's conversion.  It holds
none of the quantization method's arithmetic.

The pages train on real model weights and activations (Qwen3.5-9B,
DS-R1-Distill-Llama-8B and others, "Key findings" of the QATFactory project
page), which are not available here; these distributions stand in for them:

* weights: N(0, std) with a fraction of entries, chosen without replacement,
  multiplied by an outlier factor;
* Q4_K weights: N(0, std) times a per-row factor exp(U(ln 0.5, ln 2));
* activations: Student-t with 3 degrees of freedom (Z / sqrt(chi2_3 / 3)), with
  a fraction of hidden channels, chosen without replacement, scaled up;
* upstream gradients: N(0, 1e-3).

Every tensor gets its own stream ``default_rng([seed, index])`` so a tensor
does not change when another one is added or resized.  ``rows_scale`` shrinks
the row count of every tensor (keeping the contiguous dimension, so blocks and
tiles stay real) for the small cases the oracle finishes in seconds.
"""
from __future__ import annotations

import numpy as np
import torch


def _rng(seed: int, index: int) -> np.random.Generator:
    return np.random.default_rng([seed, index])


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """FP32 samples -> BF16 (torch's round-to-nearest-even conversion)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _out(a: np.ndarray, dtype: str) -> torch.Tensor:
    """BF16 tensor, or the FP32 samples themselves (latent master weights)."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return to_bf16(a)


def normal_with_outliers(rows: int, cols: int, std: float, frac: float, factor: float,
                         seed: int, index: int = 0, dtype: str = "bf16") -> torch.Tensor:
    rng = _rng(seed, index)
    a = rng.standard_normal(rows * cols, dtype=np.float32) * np.float32(std)
    k = int(round(frac * a.size))
    if k:
        idx = rng.choice(a.size, size=k, replace=False)
        a[idx] *= np.float32(factor)
    return _out(a.reshape(rows, cols), dtype)


def row_scaled_normal(rows: int, cols: int, std: float, lo: float, hi: float,
                      seed: int, index: int = 0, dtype: str = "bf16") -> torch.Tensor:
    rng = _rng(seed, index)
    a = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    f = np.exp(rng.uniform(np.log(lo), np.log(hi), size=(rows, 1))).astype(np.float32)
    return _out(a * f, dtype)


def student_t_channels(rows: int, cols: int, df: float, chan_frac: float, factor: float,
                       seed: int, index: int = 0) -> torch.Tensor:
    rng = _rng(seed, index)
    z = rng.standard_normal((rows, cols), dtype=np.float32)
    chi2 = rng.standard_gamma(df / 2.0, size=(rows, cols), dtype=np.float32) * np.float32(2.0)
    a = z / np.sqrt(chi2 / np.float32(df))
    k = int(round(chan_frac * cols))
    if k:
        ch = rng.choice(cols, size=k, replace=False)
        a[:, ch] *= np.float32(factor)
    return to_bf16(a)


def _rows(r: int, rows_scale: float) -> int:
    return max(1, int(round(r * rows_scale)))


# --------------------------------------------------------------------------
# The five workloads.  Each returns a dict with the tensors and their roles.
# --------------------------------------------------------------------------
def nvfp4_weight(rows_scale: float = 1.0, seed: int = 0):
    """NVFP4 weight fake-quant of one BF16 4096x4096 matrix, N(0, 0.02) with
    0.1% of entries scaled x20."""
    w = normal_with_outliers(_rows(4096, rows_scale), 4096, 0.02, 1e-3, 20.0, seed, 0)
    return {"tensors": [w], "names": ["w"], "groups": [0], "n_groups": 1}


def mxfp4_w4a4(rows_scale: float = 1.0, seed: int = 1):
    """MXFP4 W4A4: weight 12288x4096 N(0, 0.02); activations 8 x 4096 tokens by
    4096 hidden, Student-t(3), 1% of hidden channels scaled x50."""
    w = normal_with_outliers(_rows(12288, rows_scale), 4096, 0.02, 0.0, 1.0, seed, 0)
    a = student_t_channels(_rows(8 * 4096, rows_scale), 4096, 3.0, 0.01, 50.0, seed, 1)
    return {"tensors": [w, a], "names": ["w", "a"], "groups": [0, 0], "n_groups": 1}


def q4k_weights(rows_scale: float = 1.0, seed: int = 2, dtype: str = "bf16"):
    """Q4_K weight-only: down-proj 4096x14336 and up-proj 14336x4096,
    N(0, 0.015) times a per-row factor log-uniform in [0.5, 2]."""
    down = row_scaled_normal(_rows(4096, rows_scale), 14336, 0.015, 0.5, 2.0, seed, 0, dtype)
    up = row_scaled_normal(_rows(14336, rows_scale), 4096, 0.015, 0.5, 2.0, seed, 1, dtype)
    return {"tensors": [down, up], "names": ["down", "up"], "groups": [0, 0], "n_groups": 1}


def nvfp4_tied(rows_scale: float = 1.0, seed: int = 3, with_grads: bool = True,
               dtype: str = "bf16"):
    """NVFP4 tied-scale fused projections: Q 4096x4096, K and V 1024x4096 (tie
    group 0), gate and up 14336x4096 (tie group 1); N(0, 0.02) with 0.1% x20
    outliers; upstream gradients N(0, 1e-3) of the same shapes.  dtype="f32" gives the FP32
    latent master weights (the same samples, not rounded to BF16)."""
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (14336, 4096), (14336, 4096)]
    names = ["q", "k", "v", "gate", "up"]
    ts = [normal_with_outliers(_rows(r, rows_scale), c, 0.02, 1e-3, 20.0, seed, i, dtype)
          for i, (r, c) in enumerate(shapes)]
    out = {"tensors": ts, "names": names, "groups": [0, 0, 0, 1, 1], "n_groups": 2}
    if with_grads:
        out["grads"] = [normal_with_outliers(t.shape[0], t.shape[1], 1e-3, 0.0, 1.0, seed,
                                             100 + i) for i, t in enumerate(ts)]
    return out


def moe_experts(n_experts: int = 128, rows_scale: float = 1.0, seed: int = 4):
    """MoE sweep: per expert gate and up 768x2048 and down 2048x768, N(0, 0.02).
    NVFP4 tie groups: {gate, up} of expert e is group 2e, {down} is 2e+1."""
    ts, names, groups = [], [], []
    for e in range(n_experts):
        for j, (nm, (r, c)) in enumerate([("gate", (768, 2048)), ("up", (768, 2048)),
                                          ("down", (2048, 768))]):
            ts.append(normal_with_outliers(_rows(r, rows_scale), c, 0.02, 0.0, 1.0, seed,
                                           3 * e + j))
            names.append(f"e{e}.{nm}")
            groups.append(2 * e + (1 if nm == "down" else 0))
    return {"tensors": ts, "names": names, "groups": groups, "n_groups": 2 * n_experts}


def nvfp4_activation(rows_scale: float = 1.0, seed: int = 5):
    """NVFP4 activation fake-quant of a 1 x 32768 x 4096 BF16 Student-t(3)
    sequence; the tracked amax starts at 0."""
    a = student_t_channels(_rows(32768, rows_scale), 4096, 3.0, 0.0, 1.0, seed, 0)
    return {"tensors": [a], "names": ["act"], "groups": [0], "n_groups": 1}


def q4k_ste_ends(seed: int = 51) -> torch.Tensor:
    """One BF16 Q4_K super-block [1, 256] whose values put elements exactly on both ends
    of the clipped STE's range [0, 15]: sub-block 0 spans -2^-8 .. 944 * 2^-8 (so its
    scale is 63 * 2^-8 and d = 2^-8), sub-block 1 peaks at 1.875 = 15 * 2^-3 (sc = 32,
    scale 2^-3), and sub-block 2's minimum is -65 * 2^-20 (= dmin, m = 1).  Element 32
    scales to 15 exactly, element 64 to 0 exactly, element 1 below 0."""
    rng = _rng(seed, 0)
    x = np.zeros(256, np.float64)
    x[0:32] = rng.uniform(0, 3.6, 32)
    x[0], x[1] = 944 * 2.0 ** -8, -2.0 ** -8
    x[32:64] = rng.uniform(0, 1.8, 32)
    x[32] = 1.875
    x[64:96] = rng.uniform(0, 0.5, 32)
    x[64] = -65 * 2.0 ** -20
    x[96:] = rng.uniform(0, 1.0, 160)
    return to_bf16(x.reshape(1, 256))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a CPU BF16 tensor as a numpy uint16 array of bit patterns."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
