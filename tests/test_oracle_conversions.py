"""Pins for the oracle's number-format conversions (CPU only).

Each conversion is checked against something other than the oracle itself:
library conversions with round-to-nearest-even semantics (ml_dtypes, numpy),
brute-force nearest-value search over the format's value set, and math.frexp.
"""
import math

import ml_dtypes
import numpy as np
import pytest

import oracle


def f32(bits):
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


def finite_f32_boundary_patterns(hi_bits: np.ndarray, shift: int) -> np.ndarray:
    """For each value of a narrower format given by its top bits, the binary32
    patterns at and around its rounding boundaries."""
    lows = np.array([0, 1, (1 << (shift - 1)) - 1, 1 << (shift - 1), (1 << (shift - 1)) + 1,
                     (1 << shift) - 1], dtype=np.uint32)
    pats = (hi_bits.astype(np.uint32)[:, None] << shift) | lows[None, :]
    pats = pats.reshape(-1)
    v = f32(pats)
    return pats[np.isfinite(v)]


# ----------------------------------------------------------------------------- BF16
def test_bf16_matches_ml_dtypes_at_every_boundary():
    pats = finite_f32_boundary_patterns(np.arange(1 << 16, dtype=np.uint32), 16)
    x = f32(pats)
    ref = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    got = oracle.f32_to_bf16(x)
    assert np.array_equal(got, ref)


def test_bf16_random_patterns():
    rng = np.random.default_rng(11)
    pats = rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x = f32(pats)
    x = x[np.isfinite(x)]
    assert np.array_equal(oracle.f32_to_bf16(x), x.astype(ml_dtypes.bfloat16).view(np.uint16))


# ----------------------------------------------------------------------------- FP16
def test_f16_matches_numpy_at_every_boundary():
    # all FP16 values as binary32, and the binary32 neighbours of every midpoint
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    hv = h.view(np.float16).astype(np.float32)
    hv = hv[np.isfinite(hv)]
    hv = np.sort(np.unique(hv))
    mids = ((hv[:-1].astype(np.float64) + hv[1:].astype(np.float64)) / 2).astype(np.float32)
    mb = mids.view(np.uint32)
    near = np.concatenate([mb - 1, mb, mb + 1]).view(np.float32)
    x = np.concatenate([hv, near, np.float32([65519.0, 65520.0, 65536.0, 1e-8, 2.0**-25,
                                              2.0**-24 * 1.5, 3e-5, 6.1e-5])])
    x = x[np.isfinite(x)]
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f32_to_f16(x), ref)


def test_f16_decode_matches_numpy():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_f32(int(v)) for v in h[::7]], dtype=np.float32)
    r = ref[::7]
    both_nan = np.isnan(got) & np.isnan(r)
    assert np.array_equal(got[~both_nan], r[~both_nan])


# ----------------------------------------------------------------------------- E2M1
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def brute_force_e2m1(q: np.ndarray) -> np.ndarray:
    """Nearest E2M1 magnitude by exhaustive search, ties to the even code,
    saturating at 6; the sign bit follows the input's sign bit."""
    a = np.abs(q.astype(np.float64))
    dist = np.abs(a[:, None] - E2M1_GRID[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among equally near codes prefer the even one (the code index is the magnitude code)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    idx = np.where(a > 6.0, 7, idx)
    sign = (q.view(np.uint32) >> 31).astype(np.uint8)
    return (sign << 3) | idx.astype(np.uint8)


def test_e2m1_matches_ml_dtypes_and_brute_force():
    rng = np.random.default_rng(3)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    mb = mids.view(np.uint32)
    special = np.concatenate([mids, (mb - 1).view(np.float32), (mb + 1).view(np.float32),
                              E2M1_GRID.astype(np.float32),
                              np.float32([6.5, 7.0, 7.99, 8.0, 1e30, 3.4e38, 1e-40, 0.0])])
    special = np.concatenate([special, -special])
    rnd = (rng.standard_normal(1_000_000) * 3).astype(np.float32)
    wide = f32(rng.integers(0, 1 << 32, 500_000, dtype=np.uint64).astype(np.uint32))
    x = np.concatenate([special, rnd, wide[np.isfinite(wide)]])
    got = oracle.e2m1_from_f32(x)
    assert np.array_equal(got, brute_force_e2m1(x))
    # library conversion (RNE, saturating); compare magnitudes and the sign of the value
    lib = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    dec = np.array([oracle.e2m1_to_f32(c) for c in range(16)], dtype=np.float32)[got]
    assert np.array_equal(dec.view(np.uint32), lib.view(np.uint32))


def test_e2m1_decode_table():
    vals = [oracle.e2m1_to_f32(c) for c in range(16)]
    assert vals[:8] == list(E2M1_GRID)
    assert vals[8:] == [-v for v in E2M1_GRID]
    assert math.copysign(1.0, vals[8]) == -1.0


def test_e2m1_exhaustive_change_points():
    """Every binary32 pattern in [0.125, 8] (where every rounding decision lies):
    the result changes exactly at the E2M1 midpoints, with ties to even."""
    lo = int(np.float32(0.125).view(np.uint32))
    hi = int(np.float32(8.0).view(np.uint32))
    pos, val, n = oracle.change_points("e2m1", lo, hi)
    # expected: code 0 from 0.125; ties at 0.25 go to 0 -> change just above 0.25, etc.
    def up(v):
        return int(np.float32(v).view(np.uint32)) + 1
    expect = [(lo, 0), (up(0.25), 1), (int(np.float32(0.75).view(np.uint32)), 2),
              (up(1.25), 3), (int(np.float32(1.75).view(np.uint32)), 4), (up(2.5), 5),
              (int(np.float32(3.5).view(np.uint32)), 6), (up(5.0), 7)]
    assert n == len(expect)
    assert [(int(p), int(v)) for p, v in zip(pos, val)] == expect


# ----------------------------------------------------------------------------- E4M3
def e4m3_value_set():
    """The 127 finite non-negative E4M3 values, decoded by ml_dtypes."""
    b = np.arange(0, 127, dtype=np.uint8)
    return b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def brute_force_e4m3(v: np.ndarray) -> np.ndarray:
    vals = e4m3_value_set()
    a = np.abs(v.astype(np.float64))
    out = np.empty(a.shape, np.uint8)
    for i in range(0, a.size, 100_000):
        ai = a[i:i + 100_000]
        dist = np.abs(ai[:, None] - vals[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        even = cand & (np.arange(127)[None, :] % 2 == 0)
        idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        idx = np.where(ai > 448.0, 126, idx)
        out[i:i + 100_000] = idx
    sign = (v.view(np.uint32) >> 31).astype(np.uint8) << 7
    return out | sign


def test_e4m3_matches_brute_force_and_ml_dtypes():
    rng = np.random.default_rng(5)
    vals = e4m3_value_set().astype(np.float32)
    mids = ((e4m3_value_set()[:-1] + e4m3_value_set()[1:]) / 2).astype(np.float32)
    mb = mids.view(np.uint32)
    special = np.concatenate([vals, mids, (mb - 1).view(np.float32), (mb + 1).view(np.float32),
                              np.float32([448, 449, 463.9, 464, 464.1, 480, 1e5, 2.0**-10,
                                          2.0**-10 * 1.0001, 1e-30, 0.0])])
    rnd = np.exp(rng.uniform(np.log(1e-4), np.log(600), 400_000)).astype(np.float32)
    x = np.concatenate([special, rnd, -rnd[:1000]])
    got = oracle.e4m3_from_f32(x)
    assert np.array_equal(got, brute_force_e4m3(x))
    inrange = np.abs(x) < 464
    lib = x[inrange].astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got[inrange], lib)
    assert np.all(got[~inrange] & 0x7F == 0x7E)          # saturates to 448


def test_e4m3_decode_matches_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    ref = b.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    got = np.array([oracle.e4m3_to_f32(int(c)) for c in b], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_e4m3_exhaustive_change_points():
    """Every binary32 pattern in [2^-11, 512]: one change per E4M3 value, at its
    lower midpoint (inclusive when that value's mantissa is even)."""
    lo = int(np.float32(2.0 ** -11).view(np.uint32))
    hi = int(np.float32(512.0).view(np.uint32))
    pos, val, n = oracle.change_points("e4m3", lo, hi)
    vals = e4m3_value_set()
    expect = [(lo, 0)]
    for code in range(1, 127):
        mid = np.float32((vals[code - 1] + vals[code]) / 2)
        mbits = int(mid.view(np.uint32))
        expect.append((mbits if code % 2 == 0 else mbits + 1, code))
    assert n == len(expect)
    assert [(int(p), int(v)) for p, v in zip(pos, val)] == expect


# ----------------------------------------------------------------------------- E8M0 exponent
def test_mx_exponent_matches_frexp_for_every_bf16():
    h = np.arange(1, 0x7F80, dtype=np.uint32)            # all positive finite BF16 values
    v = f32(h << 16)
    for x in v[::3]:
        m, k = math.frexp(float(x))
        want = max(-127, min(127, (k - 1) - 2))
        assert oracle.mx_exponent(float(x)) == want
    assert oracle.mx_exponent(0.0) == -127
    # E8M0 byte e+127 decodes (ml_dtypes) to 2^e
    for e in (-127, -3, 0, 5, 125):
        byte = np.uint8(e + 127)
        assert float(np.array([byte]).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)[0]) == 2.0 ** e


def test_conversions_are_monotone_in_magnitude():
    """Every oracle conversion is a non-decreasing step function of the binary32 bit
    pattern within one sign (round-to-nearest is monotone); the exhaustive GPU check
    of the hardware conversions relies on this."""
    rng = np.random.default_rng(8)
    pats = np.unique(np.concatenate([
        rng.integers(0, 0x7F7FFFFF, 1_000_000, dtype=np.uint64).astype(np.uint32),
        np.arange(0x3E000000, 0x3E000000 + 200_000, dtype=np.uint32)]))
    for sign in (0, 0x80000000):
        x = (pats | np.uint32(sign)).view(np.float32)
        for conv, mask in ((oracle.e2m1_from_f32, 0x7), (oracle.e4m3_from_f32, 0x7F),
                           (oracle.f32_to_bf16, 0x7FFF), (oracle.f32_to_f16, 0x7FFF)):
            m = (conv(x).astype(np.int64)) & mask
            assert np.all(np.diff(m) >= 0)
