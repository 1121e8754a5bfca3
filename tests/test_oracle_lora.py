"""Pins for the oracle's LoRA merge (CPU only).

LoRA-QAD (QATFactory project page, Method, "QAD") trains low-rank adapters on a
frozen BF16 base and quantizes the merged weight W + scale * B A.  The oracle
materializes the merge in BF16 with B A accumulated in FP32 in increasing k.
"""
import ml_dtypes
import numpy as np
import torch

import oracle
import workloads


def bf16(a):
    return np.ascontiguousarray(np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16))


def f32(h):
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def test_exact_integer_grid_merge_matches_numpy():
    """Small integers times powers of two: every product and partial sum is exact in
    FP32, so the merge equals the exact W + scale*(B @ A), rounded once to BF16."""
    rng = np.random.default_rng(1)
    rows, cols, r = 24, 96, 16
    b = rng.integers(-8, 9, (rows, r)).astype(np.float32) * np.float32(2.0 ** -6)
    a = rng.integers(-8, 9, (r, cols)).astype(np.float32) * np.float32(2.0 ** -5)
    w = rng.integers(-64, 65, (rows, cols)).astype(np.float32) * np.float32(2.0 ** -7)
    scale = 0.5
    exact = w.astype(np.float64) + scale * (b.astype(np.float64) @ a.astype(np.float64))
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)   # exact in FP32
    want = bf16(exact.astype(np.float32))
    got = oracle.lora_merge(bf16(w), bf16(b), bf16(a), scale)
    assert np.array_equal(got, want)


def test_zero_adapter_or_scale_gives_the_base():
    w = workloads.bf16_bits(workloads.normal_with_outliers(8, 64, 0.02, 0.01, 20, 3, 0))
    w[0, 0] = 0x8000                                             # a negative zero
    b = bf16(np.random.default_rng(2).standard_normal((8, 4)))
    a = bf16(np.random.default_rng(3).standard_normal((4, 64)))
    for bb, s in ((np.zeros_like(b), 1.0), (b, 0.0)):
        m = oracle.lora_merge(w, bb, a, s)
        keep = w != 0x8000
        assert np.array_equal(m[keep], w[keep])
        assert m[0, 0] == 0x0000                                # -0 + +0 = +0


def test_random_merge_within_one_bf16_step_of_float64():
    rng = np.random.default_rng(4)
    rows, cols, r = 32, 256, 16
    w = workloads.bf16_bits(workloads.normal_with_outliers(rows, cols, 0.02, 1e-3, 20, 5, 0))
    b = bf16(rng.standard_normal((rows, r)) * 0.01)
    a = bf16(rng.standard_normal((r, cols)) * 0.02)
    scale = 2.0
    ref = f32(w).astype(np.float64) + scale * (f32(b).astype(np.float64) @ f32(a).astype(np.float64))
    got = f32(oracle.lora_merge(w, b, a, scale)).astype(np.float64)
    # one BF16 step of the reference value
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= step)
    # and it is not the unmerged base (the adapter matters at this scale)
    assert np.mean(got != f32(w)) > 0.5


def test_merge_locality():
    rng = np.random.default_rng(6)
    rows, cols, r = 6, 64, 8
    w = bf16(rng.standard_normal((rows, cols)) * 0.1)
    b = bf16(rng.standard_normal((rows, r)))
    a = bf16(rng.standard_normal((r, cols)))
    base = oracle.lora_merge(w, b, a, 0.25)
    b2 = b.copy()
    b2[3, 5] ^= 0x0040
    m = oracle.lora_merge(w, b2, a, 0.25)
    diff_rows = np.nonzero((m != base).any(axis=1))[0]
    assert list(diff_rows) == [3]
    a2 = a.copy()
    a2[2, 17] ^= 0x0040
    m = oracle.lora_merge(w, b, a2, 0.25)
    diff_cols = np.nonzero((m != base).any(axis=0))[0]
    assert list(diff_cols) == [17]


def test_accumulation_order_is_increasing_k():
    """A hand-worked case that tells the summation orders apart.  The products
    b_k * a_k are 1, 2^-8, 2^-24, 2^-24 (each exact).
      increasing k:  1 + 2^-8 is exact; adding 2^-24 is a tie at half an FP32 ulp
                     and rounds to the even 1 + 2^-8, twice; BF16(1 + 2^-8) is again
                     a tie, to the even 1.0.
      decreasing k or the exact sum:  2^-24 + 2^-24 + 2^-8 + 1 = 1 + 2^-8 + 2^-23,
                     which BF16 rounds up to 1 + 2^-7.
    The oracle must give 1.0 (W = 0, scale = 1)."""
    b = bf16([[1.0, 2.0 ** -4, 2.0 ** -12, 2.0 ** -12]])
    a = bf16([[1.0], [2.0 ** -4], [2.0 ** -12], [2.0 ** -12]])
    w = bf16([[0.0]])
    got = f32(oracle.lora_merge(w, b, a, 1.0).astype(np.uint32))
    assert got.reshape(-1).tolist() == [1.0]
    # the same products in decreasing k reach the other side of the BF16 tie
    rev = f32(oracle.lora_merge(w, b[:, ::-1].copy(), a[::-1, :].copy(), 1.0).astype(np.uint32))
    assert rev.reshape(-1).tolist() == [1.0 + 2.0 ** -7]


def _fused_chain_reference(w, b, a, scale):
    """The merge with each term rounded once (acc + b*a), emulated in float64: every
    b*a of BF16 operands is exact in float64, and rounding acc + b*a first to binary64
    and then to binary32 equals rounding it once to binary32 (the binary64 precision is
    at least twice binary32's plus two, and both addends are binary32 values here)."""
    wf, bf, af = f32(w), f32(b), f32(a)
    rows, cols = wf.shape
    r = bf.shape[1]
    acc = np.zeros((rows, cols), np.float32)
    for k in range(r):
        prod = bf[:, k:k + 1].astype(np.float64) * af[k:k + 1, :].astype(np.float64)
        acc = (acc.astype(np.float64) + prod).astype(np.float32)
    d = (np.float32(scale) * acc).astype(np.float32)
    return bf16((wf + d).astype(np.float32))


def test_merge_is_one_rounding_per_term_on_random_adapters():
    rng = np.random.default_rng(11)
    rows, cols, r = 16, 128, 16
    w = workloads.bf16_bits(workloads.normal_with_outliers(rows, cols, 0.02, 1e-3, 20, 12, 0))
    b = bf16(rng.standard_normal((rows, r)) * 0.01)
    a = bf16(rng.standard_normal((r, cols)) * 0.02)
    got = oracle.lora_merge(w, b, a, 2.0)
    assert np.array_equal(got, _fused_chain_reference(w, b, a, 2.0))


def test_underflowing_product_is_fused_into_the_sum():
    """A worked case where a product underflows FP32.  Terms: b0*a0 = 2^-149 (the
    smallest subnormal) and b1*a1 = 2^-150.  Fused: acc = RN(2^-149 + 2^-150), a tie
    between 2^-149 and 2^-148 that goes to the even 2^-148.  Multiplying first would
    round 2^-150 to 0 (a tie, to even) and leave acc = 2^-149.  With W = 0 and
    scale = 2^100 the merged weight is 2^-48 (0x2780) fused, 2^-49 (0x2700) if not."""
    w = np.zeros((1, 2), np.uint16)
    b = bf16(np.float32([[2.0 ** -75, 2.0 ** -75]] * 1))
    a = bf16(np.float32([[2.0 ** -74, 2.0 ** -74], [2.0 ** -75, 2.0 ** -75]]))
    got = oracle.lora_merge(w, b, a, 2.0 ** 100)
    assert got.tolist() == [[0x2780, 0x2780]]
