"""The bounds the merged-weight amax kernel (k_lora_amax) prunes with, checked on the CPU.

For the merged weight M = BF16(W + RN(s * acc)), acc the fused FP32 sum of b_k a_k,
the kernel uses, per element (row i, column j),
    K_i = RN(RN(|s| * R_i) * (1 + 2^-6)),  R_i = FP32 sum of |b_ik| in increasing k
    D   = RN(RN(K_i * C_j) + tiny),  tiny = RN(2^-120 + RN(|s| * 2^-140)),  C_j = max_k |a_kj|
          (D = 0 when K_i or C_j is 0)
    ub  = RN(RN(|W| + D) * (1 + 2^-7))
    lb  = RN(RN(RN(|W| - D) * (1 - 2^-7)) - 2^-120)
and relies on lb <= |M| <= ub.  Here both sides are computed in binary32 exactly as the
kernel rounds them (numpy float32 operations round to nearest even) and |M| comes from
the oracle's merge, over random adapters, outliers, subnormal and huge values."""
import zlib

import numpy as np
import pytest

import oracle


def f32(h):
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def bf16(a):
    import ml_dtypes
    return np.ascontiguousarray(np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16))


def kernel_bounds(w, b, a, s):
    W, B, A = f32(w), f32(b), f32(a)
    F = np.float32
    sabs = F(abs(s))
    R = np.zeros(B.shape[0], F)
    for k in range(B.shape[1]):
        R = (R + np.abs(B[:, k])).astype(F)
    K = ((sabs * R).astype(F) * F(1 + 2.0 ** -6)).astype(F)
    C = np.abs(A).max(axis=0).astype(F)
    tiny = (F(2.0 ** -120) + (sabs * F(2.0 ** -140)).astype(F)).astype(F)
    KC = (K[:, None] * C[None, :]).astype(F)
    D = np.where((K[:, None] > 0) & (C[None, :] > 0), (KC + tiny).astype(F), F(0))
    x = np.abs(W)
    ub = ((x + D).astype(F) * F(1 + 2.0 ** -7)).astype(F)
    lb = (((x - D).astype(F) * F(1 - 2.0 ** -7)).astype(F) - F(2.0 ** -120)).astype(F)
    return lb, ub


CASES = [
    ("normal", 0.02, 0.01, 0.02, 2.0),
    ("outliers", 0.5, 0.01, 0.02, 2.0),
    ("merge_dominates", 1e-6, 0.3, 0.3, 4.0),
    ("subnormal", 1e-38, 1e-20, 1e-19, 1.0),
    ("tiny_products", 1e-3, 1e-25, 1e-20, 2.0 ** 60),
    ("huge", 1e30, 1e14, 1e14, 2.0 ** 10),
    ("odd_scale", 0.02, 0.01, 0.02, -0.3),
]


@pytest.mark.parametrize("name,ws,bs,as_,s", CASES)
def test_bounds_hold(name, ws, bs, as_, s):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    rows, cols, r = 48, 96, 16
    w = bf16(rng.standard_normal((rows, cols)) * ws)
    b = bf16(rng.standard_normal((rows, r)) * bs)
    a = bf16(rng.standard_normal((r, cols)) * as_)
    m = np.abs(f32(oracle.lora_merge(w, b, a, s)))
    lb, ub = kernel_bounds(w, b, a, s)
    finite = np.isfinite(m)
    assert np.all(m[finite] <= ub[finite]), name
    assert np.all(lb[finite] <= m[finite]), name


def test_zero_adapter_bounds_are_exact():
    """With B = 0 every product is an exact zero: D = 0, so ub = |W|(1 + 2^-7) and the
    merge gives M = W exactly."""
    rng = np.random.default_rng(3)
    w = bf16(rng.standard_normal((8, 32)) * 0.02)
    b = np.zeros((8, 4), np.uint16)
    a = bf16(rng.standard_normal((4, 32)))
    m = oracle.lora_merge(w, b, a, 2.0)
    assert np.array_equal(m & 0x7FFF, w & 0x7FFF)
    lb, ub = kernel_bounds(w, b, a, 2.0)
    assert np.all(lb <= np.abs(f32(m))) and np.all(np.abs(f32(m)) <= ub)


def test_margins_are_needed_where_the_bound_is_tight():
    """Rank 1 with b = 1 and a below one BF16 unit of W: the Holder bound is then tight
    (|acc| = |b||a| = R C exactly) and the BF16 rounding of W + s*acc often lands above
    |W| + |s*acc|.  Without the relative margins the upper bound fails on such elements;
    the kernel's bounds hold on every one."""
    rng = np.random.default_rng(11)
    rows, cols = 64, 256
    w = bf16(rng.uniform(1.0, 2.0, (rows, cols)))
    b = bf16(np.ones((rows, 1)))
    a = bf16(rng.uniform(0.0, 2.0 ** -7, (1, cols)))
    m = np.abs(f32(oracle.lora_merge(w, b, a, 1.0)))
    lb, ub = kernel_bounds(w, b, a, 1.0)
    assert np.all(m <= ub) and np.all(lb <= m)
    plain = np.abs(f32(w)) + np.abs(f32(a))          # |W| + |s*acc| with no margin
    assert np.count_nonzero(m > plain) > 0
