"""Pins for the oracle's MSE-searched Q4_K fit (CPU only).

The project page's "Key findings" use an MSE-optimal quantizer as the Q4_K PTQ
baseline without giving its steps.  The oracle's reading: with the sub-block's
offset fixed by its minimum, search the scale (hi + min_j) / n over
n in {15, 14, 14.5, 15.5, 16, 16.5, 17, 17.5, 18} for the least squared error.
"""
import numpy as np

import oracle
import workloads

GRID = [15.0, 14.0, 14.5, 15.5, 16.0, 16.5, 17.0, 17.5, 18.0]


def err64(v, scale, m):
    v = v.astype(np.float64)
    q = np.clip(np.round((v + m) / scale), 0, 15)      # round half even, like RNE
    return float(np.sum((v - (scale * q - m)) ** 2))


def subblocks(t):
    x = t.float().numpy().reshape(-1, 32)
    return x


def test_search_picks_a_grid_scale_with_least_error():
    wl = workloads.q4k_weights(rows_scale=1 / 256)
    x = np.concatenate([subblocks(t) for t in wl["tensors"]])[:4000]
    rng = np.random.default_rng(0)
    x = np.concatenate([x, rng.standard_t(3, (500, 32)).astype(np.float32) * 0.02])
    improved = 0
    for v in x:
        hi, mn = float(v.max()), float(v.min())
        m = -mn if mn < 0 else 0.0
        s = oracle.q4k_search_scale(v, hi, m)
        rng_ = np.float32(np.float32(hi) + np.float32(m))
        cands = [np.float32(rng_ / np.float32(n)) for n in GRID]
        assert any(s == c for c in cands)                  # one of the grid's scales
        e = [err64(v, float(c), m) for c in cands]
        es = err64(v, s, m)
        assert es <= min(e) * (1 + 1e-5) + 1e-20           # the least error on the grid
        assert es <= e[0] * (1 + 1e-5) + 1e-20             # never worse than min/max
        improved += s != cands[0]
    assert improved > len(x) // 4                           # the search does move the scale


def test_on_grid_blocks_keep_the_min_max_fit():
    # a sub-block already on a 15-step grid has zero error at n = 15, so it stays
    v = (np.arange(32) % 16).astype(np.float32) * np.float32(0.125) - np.float32(0.5)
    v = v.astype(np.float32)
    s = oracle.q4k_search_scale(v, float(v.max()), 0.5)
    assert s == np.float32(np.float32(v.max() + 0.5) / np.float32(15.0))


def test_equal_errors_keep_the_earlier_trial():
    """Trials are taken in the order 15, 14, 14.5, ... and a later one must be strictly
    better.  A two-valued sub-block {0, 210 * 2^-10} (210 = 14 * 15) is exact on both
    the n = 15 grid (scale 14 * 2^-10) and the n = 14 grid (scale 15 * 2^-10): both
    errors are 0, every other trial's is positive, and the search keeps n = 15."""
    hi = np.float32(210 * 2.0 ** -10)
    rng = np.random.default_rng(61)
    v = np.where(rng.random(32) < 0.5, np.float32(0), hi).astype(np.float32)
    v[0], v[1] = 0, hi
    cands = [np.float32(hi / np.float32(n)) for n in GRID]
    errs = [err64(v, float(c), 0.0) for c in cands]
    assert errs[0] == 0 and errs[1] == 0 and min(errs[2:]) > 0
    assert oracle.q4k_search_scale(v, float(hi), 0.0) == cands[0]


def test_mse_fit_decoder_and_total_error():
    wl = workloads.q4k_weights(rows_scale=1 / 256)
    tot_mm = tot_mse = 0.0
    for t in wl["tensors"]:
        y, b = oracle.q4k(t, mse=True)
        assert np.array_equal(oracle.q4k_decode(b, y.size), y)
        y0, _ = oracle.q4k(t)
        x = t.float().numpy().reshape(-1).astype(np.float64)
        tot_mse += float(np.sum((oracle.bf16_to_f32(y).astype(np.float64) - x) ** 2))
        tot_mm += float(np.sum((oracle.bf16_to_f32(y0).astype(np.float64) - x) ** 2))
    assert tot_mse < 0.97 * tot_mm                          # a visibly better fit


def test_mse_fit_equals_min_max_fit_on_grid_superblocks():
    """Sub-blocks whose values sit exactly on their 15-step min/max grid have zero
    error at n = 15, so the search keeps the min/max scale: both fits agree."""
    rng = np.random.default_rng(21)
    for _ in range(20):
        vals = []
        for j in range(8):
            s = 2.0 ** int(rng.integers(-9, -4))
            m = s * int(rng.integers(0, 16))
            q = rng.integers(0, 16, 32)
            q[:2] = [0, 15]
            vals.append((q * s - m).astype(np.float32))
        x = np.concatenate(vals)
        xb = (x.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal((xb.astype(np.uint32) << 16).view(np.float32), x)   # exact BF16
        a = oracle.q4k_fit_one(xb, mse=False)
        b = oracle.q4k_fit_one(xb, mse=True)
        assert a[0] == b[0] and a[1] == b[1]
        for u, v in zip(a[2:], b[2:]):
            assert np.array_equal(u, v)
