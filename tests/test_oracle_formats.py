"""Pins for the oracle's NVFP4 / MXFP4 / Q4_K quantize-dequantize, pack, tied
amax and STE (CPU only).

What the QATFactory pages fix ("Supported formats" table; Method, "Numerics")
is checked directly: block sizes, bits per weight, symmetric vs asymmetric,
the tied NVFP4 tensor scale.  Everything the pages leave open is pinned by
properties that a wrong term, sign, index or operand would break: exact round
trips of values already on the grid, brute-force nearest-code search, an
independent decoder, locality of blocks, symmetry and idempotence.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "format_table.json")
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bits_of(a: np.ndarray) -> np.ndarray:
    """FP32 values that are exactly BF16 -> BF16 bit patterns (asserting exactness)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = a.view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "value not exactly representable in BF16"
    return (b >> 16).astype(np.uint16)


def f32_of(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32)


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    out = np.empty(codes.size * 2, np.uint8)
    out[0::2] = codes & 15
    out[1::2] = codes >> 4
    return out


def e2m1_val(c: np.ndarray) -> np.ndarray:
    v = E2M1[c & 7]
    return np.where(c & 8, -v, v)


def rand_bf16(rows, cols, seed, std=0.02):
    return workloads.normal_with_outliers(rows, cols, std, 1e-3, 20.0, seed, 0)


# ----------------------------------------------------------------------------- bits per weight
def test_bits_per_weight_and_block_sizes_match_format_table():
    table = json.load(open(GOLDEN))
    rows, cols = 3, 512
    x = rand_bf16(rows, cols, 1)
    n = rows * cols
    y, codes, scales, st = oracle.nvfp4(x, oracle.amax(x))
    assert n // scales.size == table["nvfp4"]["block"]
    assert (codes.nbytes + scales.nbytes) * 8 / n == table["nvfp4"]["bits_per_weight"]
    y, codes, scales = oracle.mxfp4(x)
    assert n // scales.size == table["mxfp4"]["block"]
    assert (codes.nbytes + scales.nbytes) * 8 / n == table["mxfp4"]["bits_per_weight"]
    y, blocks = oracle.q4k(x)
    assert blocks.size // 144 == n // table["q4k"]["superblock"]
    assert blocks.nbytes * 8 / n == table["q4k"]["bits_per_weight"]


# ----------------------------------------------------------------------------- tied scale
def test_tied_tensor_scale_is_amax_of_concatenation():
    """NVFP4: projections an engine fuses (QKV, gate/up) use a common tensor scale (Method, Numerics)."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False)
    am = oracle.tied_amax(wl["tensors"], wl["groups"], wl["n_groups"])
    for g in range(2):
        cat = np.concatenate([t.float().numpy().reshape(-1) for t, gg in
                              zip(wl["tensors"], wl["groups"]) if gg == g])
        assert am[g] == np.abs(cat).max()
        st = oracle.nvfp4_tensor_scale(am[g])
        assert st == np.float32(np.abs(cat).max()) / np.float32(2688.0)
        # every tensor of the group is quantized with that same scale
        for t, gg in zip(wl["tensors"], wl["groups"]):
            if gg == g:
                assert oracle.nvfp4(t, am[g])[3] == st
    tracked = np.float32([1e9, 0.0])
    am2 = oracle.tied_amax(wl["tensors"], wl["groups"], 2, tracked=tracked)
    assert am2[0] == np.float32(1e9) and am2[1] == am[1]


# ----------------------------------------------------------------------------- on-grid round trips
def make_nvfp4_on_grid(rows, cols, seed, k=-9):
    """x = code * sb * s_t with s_t = 2^k, E4M3 sb, every block holding a +-6 and
    one block using sb = 448, so the fit must recover every code and scale."""
    rng = np.random.default_rng(seed)
    nb = rows * cols // 16
    st = np.float32(2.0 ** k)
    sb = rng.integers(0x08, 0x7F, size=nb).astype(np.uint8)   # normal E4M3, <= 448
    sb[rng.integers(nb)] = 0x7E                                 # 448 somewhere
    sbv = sb.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    codes = rng.integers(0, 16, size=(nb, 16)).astype(np.uint8)
    codes[np.arange(nb), rng.integers(0, 16, nb)] = 7 | (rng.integers(0, 2, nb) << 3).astype(np.uint8)
    x = (e2m1_val(codes) * sbv[:, None] * st).astype(np.float32)
    return bits_of(x.reshape(rows, cols)), codes.reshape(-1), sb, st


def test_nvfp4_round_trip_of_on_grid_values():
    xb, codes, sb, st = make_nvfp4_on_grid(8, 256, 7)
    am = oracle.amax(xb)
    assert am == np.float32(2688.0) * st
    y, c, s, st_out = oracle.nvfp4(xb, am)
    assert st_out == st
    assert np.array_equal(y, xb.reshape(-1))
    assert np.array_equal(s, sb)
    assert np.array_equal(unpack_nibbles(c), codes)


def test_mxfp4_round_trip_of_on_grid_values():
    rng = np.random.default_rng(9)
    rows, cols = 6, 320
    nb = rows * cols // 32
    e = rng.integers(-120, 120, nb)
    codes = rng.integers(0, 16, size=(nb, 32)).astype(np.uint8)
    top = rng.choice([6, 7], nb).astype(np.uint8) | (rng.integers(0, 2, nb) << 3).astype(np.uint8)
    codes[np.arange(nb), rng.integers(0, 32, nb)] = top       # block max 4*2^e or 6*2^e
    x = (e2m1_val(codes) * np.exp2(e.astype(np.float64))[:, None]).astype(np.float32)
    xb = bits_of(x.reshape(rows, cols))
    y, c, s = oracle.mxfp4(xb)
    assert np.array_equal(y, xb.reshape(-1))
    assert np.array_equal(s.astype(np.int64), e + 127)
    assert np.array_equal(unpack_nibbles(c), codes.reshape(-1))


def _bf16_exact_int(v: int) -> bool:
    """An integer times a power of two is exact in BF16 iff it has <= 8 significant bits."""
    v = abs(v)
    while v and v % 2 == 0:
        v //= 2
    return v < 256


def test_q4k_round_trip_of_on_grid_values():
    """x = d*sc*q - dmin*m on a grid the min/max fit must recover exactly: in every
    super-block one sub-block has sc = 63, another has m = 63, every sub-block has
    q = 0 and q = 15 present, and all values are exact in BF16."""
    rng = np.random.default_rng(21)
    xs, want = [], []
    while len(xs) < 24:
        a = int(rng.integers(-16, -6))
        b = a + int(rng.integers(-2, 3))            # d = 2^a, dmin = 2^b
        lo = min(a, b)
        def ival(scj, mj, q):                       # value / 2^lo as an exact integer
            return scj * q * 2 ** (a - lo) - mj * 2 ** (b - lo)
        pairs = [(s_, m_) for s_ in range(1, 64) for m_ in range(0, 64)
                 if _bf16_exact_int(ival(s_, m_, 15)) and _bf16_exact_int(ival(s_, m_, 0))]
        if not any(p[0] == 63 for p in pairs) or not any(p[1] == 63 for p in pairs):
            continue
        sc = np.empty(8, np.int64)
        m = np.empty(8, np.int64)
        for j in range(8):
            if j == 0:
                cand = [p for p in pairs if p[0] == 63]
            elif j == 1:
                cand = [p for p in pairs if p[1] == 63]
            else:
                cand = pairs
            sc[j], m[j] = cand[rng.integers(len(cand))]
        perm = rng.permutation(8)
        sc, m = sc[perm], m[perm]
        x = np.empty(256)
        q = np.empty(256, np.int64)
        for j in range(8):
            exact = [k for k in range(16) if _bf16_exact_int(ival(sc[j], m[j], k))]
            qj = rng.choice(exact, 32)
            qj[:2] = [0, 15]
            rng.shuffle(qj)
            q[32 * j:32 * j + 32] = qj
            x[32 * j:32 * j + 32] = [ival(sc[j], m[j], k) * 2.0 ** lo for k in qj]
        xs.append(x)
        want.append((2.0 ** a, 2.0 ** b, sc, m, q))
    xb = bits_of(np.concatenate(xs).reshape(3, 2048))
    for i in range(24):
        d_bits, dmin_bits, sc, m, q = oracle.q4k_fit_one(xb.reshape(-1)[256 * i:256 * i + 256])
        d, dmin, sc_w, m_w, q_w = want[i]
        assert np.float16(d).view(np.uint16) == d_bits
        assert np.float16(dmin).view(np.uint16) == dmin_bits
        mw = np.where(m_w == 0, 0, m_w)
        assert np.array_equal(sc, sc_w) and np.array_equal(m, mw) and np.array_equal(q, q_w)
    y, blocks = oracle.q4k(xb)
    assert np.array_equal(y, xb.reshape(-1))


# ----------------------------------------------------------------------------- symmetry
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_symmetric_formats_are_odd(fmt):
    x = rand_bf16(16, 512, 4)
    xn = (workloads.bf16_bits(x) ^ 0x8000).astype(np.uint16)
    if fmt == "nvfp4":
        a = oracle.nvfp4(x, oracle.amax(x))
        b = oracle.nvfp4(xn.reshape(16, 512), oracle.amax(x))
    else:
        a = oracle.mxfp4(x)
        b = oracle.mxfp4(xn.reshape(16, 512))
    assert np.array_equal(a[0] ^ 0x8000, b[0])                 # y(-x) = -y(x), bitwise
    assert np.array_equal(a[1] ^ 0x88, b[1])                   # codes differ in the sign bits only
    assert np.array_equal(a[2], b[2])                          # same scales


def test_q4k_is_not_symmetric():
    """Q4_K is asymmetric: a sub-block of positive values uses m = 0, its negation does not."""
    x = np.abs(np.random.default_rng(2).standard_normal(256)).astype(np.float32) + 0.01
    xb = bits_of((x.view(np.uint32) & 0xFFFF0000).view(np.float32))
    _, _, _, m, _ = oracle.q4k_fit_one(xb)
    _, _, _, m2, _ = oracle.q4k_fit_one(xb ^ 0x8000)
    assert np.all(m == 0) and np.all(m2 > 0)


# ----------------------------------------------------------------------------- block locality
@pytest.mark.parametrize("fmt,blk", [("nvfp4", 16), ("mxfp4", 32), ("q4k", 256)])
def test_changing_one_element_changes_only_its_block(fmt, blk):
    rows, cols = 4, 1024
    x = workloads.bf16_bits(rand_bf16(rows, cols, 8)).reshape(-1).copy()
    am = oracle.amax(x)
    i = 1000 + 7
    x2 = x.copy()
    x2[i] = np.uint16(x2[i] ^ 0x0040)                            # perturb the mantissa
    assert abs(f32_of(x2[i:i + 1])[0]) < am                    # tensor amax unchanged
    def run(v):
        v = v.reshape(rows, cols)
        if fmt == "nvfp4":
            y, c, s, _ = oracle.nvfp4(v, am)
            return y, unpack_nibbles(c), np.repeat(s, 16)
        if fmt == "mxfp4":
            y, c, s = oracle.mxfp4(v)
            return y, unpack_nibbles(c), np.repeat(s, 32)
        y, b = oracle.q4k(v)
        return y, np.repeat(b.reshape(-1, 144), 256, axis=0), None
    a, b = run(x), run(x2)
    outside = np.ones(rows * cols, bool)
    outside[(i // blk) * blk:(i // blk + 1) * blk] = False
    for u, v in zip(a, b):
        if u is None:
            continue
        assert np.array_equal(u[outside], v[outside])


# ----------------------------------------------------------------------------- brute force
def test_nvfp4_codes_and_scales_are_brute_force_nearest():
    x = rand_bf16(32, 512, 12)
    xb = workloads.bf16_bits(x).reshape(-1)
    am = oracle.amax(x)
    y, c, s, st = oracle.nvfp4(x, am)
    xf = f32_of(xb).reshape(-1, 16)
    amax_b = np.abs(xf).max(axis=1)
    # block scale: nearest E4M3 (library conversion, in range) of amax_b / (6 s_t)
    ratio = (amax_b / (np.float32(6.0) * np.float32(st))).astype(np.float32)
    assert np.all(ratio < 464)
    assert np.array_equal(s, ratio.astype(ml_dtypes.float8_e4m3fn).view(np.uint8))
    S = (s.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(st)).astype(np.float32)
    inv = np.where(S == 0, np.float32(0), np.float32(1) / S).astype(np.float32)
    q = (xf * inv[:, None]).astype(np.float32).reshape(-1)
    # brute-force nearest E2M1 of the scaled value, ties to the even code, saturating
    a = np.abs(q.astype(np.float64))
    dist = np.abs(a[:, None] - E2M1[None, :])
    cand = dist == dist.min(axis=1, keepdims=True)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    idx = np.where(a > 6, 7, idx)
    want = idx.astype(np.uint8) | ((q.view(np.uint32) >> 31).astype(np.uint8) << 3)
    assert np.array_equal(unpack_nibbles(c), want)
    # dequant: f32(code) * S, rounded to BF16 by the library
    deq = (e2m1_val(want).astype(np.float32).reshape(-1, 16) * S[:, None]).astype(np.float32)
    assert np.array_equal(y, deq.reshape(-1).astype(ml_dtypes.bfloat16).view(np.uint16))


def test_mxfp4_codes_are_brute_force_nearest():
    wl = workloads.mxfp4_w4a4(rows_scale=1 / 512)
    for t in wl["tensors"]:
        y, c, s = oracle.mxfp4(t)
        xf = f32_of(workloads.bf16_bits(t).reshape(-1)).reshape(-1, 32)
        e = s.astype(np.int64) - 127
        q = (xf.astype(np.float64) * np.exp2(-e.astype(np.float64))[:, None]).reshape(-1)
        a = np.abs(q)
        dist = np.abs(a[:, None] - E2M1[None, :])
        cand = dist == dist.min(axis=1, keepdims=True)
        even = cand & (np.arange(8)[None, :] % 2 == 0)
        idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        idx = np.where(a > 6, 7, idx)
        got = unpack_nibbles(c)
        assert np.array_equal(got & 7, idx)
        # the scale puts the block max in E2M1's top binade: 4 <= amax * 2^-e < 8
        amax_b = np.abs(xf).max(axis=1).astype(np.float64) * np.exp2(-e.astype(np.float64))
        nz = amax_b > 0
        assert np.all((amax_b[nz] >= 4) & (amax_b[nz] < 8))


def test_q4k_q_is_brute_force_nearest_and_error_bounded():
    wl = workloads.q4k_weights(rows_scale=1 / 512)
    base = workloads.bf16_bits(wl["tensors"][1]).reshape(-1)[:256 * 64]
    bf = f32_of(base)
    # zero-mean weights, plus sub-blocks of one sign (all positive / all negative)
    extra = [np.abs(bf) + np.float32(0.01), -np.abs(bf) - np.float32(0.003)]
    cases = [workloads.bf16_bits(t).reshape(-1) for t in wl["tensors"]]
    cases += [oracle.f32_to_bf16(e) for e in extra]
    for xb in cases:
        for sbi in range(0, xb.size // 256, 5):
            blk = xb[256 * sbi:256 * sbi + 256]
            d_bits, dmin_bits, sc, m, q = oracle.q4k_fit_one(blk)
            d = np.float32(np.uint16(d_bits).view(np.float16))
            dmin = np.float32(np.uint16(dmin_bits).view(np.float16))
            assert np.all(sc <= 63) and np.all(m <= 63) and np.all(q <= 15)
            xf = f32_of(blk).reshape(8, 32)
            # the 6-bit scale and min are the nearest multiples of d and dmin (capped at 63)
            # of each sub-block's range/15 and of -min(0, min x); d and dmin are the FP16
            # nearest to the largest of those over the super-block divided by 63
            rng_j = (xf.max(axis=1).astype(np.float64) - np.minimum(xf.min(axis=1), 0)) / 15
            min_j = -np.minimum(xf.min(axis=1), 0).astype(np.float64)
            assert d == np.float32(np.float16(np.float32(np.float32(rng_j.max()) / np.float32(63))))
            assert dmin == np.float32(np.float16(np.float32(np.float32(min_j.max()) / np.float32(63))))
            for val, k6, unit in ((rng_j, sc, d), (min_j, m, dmin)):
                if unit > 0:
                    capped = val / float(unit) > 63.5
                    dev = np.abs(val - float(unit) * k6.astype(np.float64))
                    assert np.all(capped | (dev <= 0.5 * float(unit) * (1 + 1e-5)))
                    assert np.all(k6[capped] == 63)
            for j in range(8):
                s = np.float32(d * np.float32(sc[j]))
                mm = np.float32(dmin * np.float32(m[j]))
                inv = np.float32(0) if s == 0 else np.float32(np.float32(1) / s)
                v = ((xf[j] + mm).astype(np.float32) * inv).astype(np.float64)
                dist = np.abs(v[:, None] - np.arange(16)[None, :])
                cand = dist == dist.min(axis=1, keepdims=True)
                even = cand & (np.arange(16)[None, :] % 2 == 0)
                idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
                assert np.array_equal(q[32 * j:32 * j + 32], idx)
                # Asymmetric uint4 over [min(0, min x), max x]: the error is at most half a
                # step, plus what the 6-bit rounding of sc (<= d/2 per step, 15 steps) and
                # of m (<= dmin/2) moves the grid's ends.
                err = np.abs(xf[j].astype(np.float64) - (float(s) * idx - float(mm)))
                bound = 0.5 * float(s) + 7.5 * float(d) + 0.5 * float(dmin)
                assert err.max() <= bound * (1 + 1e-6) + 1e-30


# ----------------------------------------------------------------------------- decoders
def test_decode_of_pack_equals_fakequant_all_formats():
    """Deployment alignment: what an engine decodes from the packed bytes is
    bitwise the forward pass's dequantized output."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 256, with_grads=False)
    am = oracle.tied_amax(wl["tensors"], wl["groups"], 2)
    for t, g in zip(wl["tensors"], wl["groups"]):
        y, c, s, st = oracle.nvfp4(t, am[g])
        assert np.array_equal(oracle.nvfp4_decode(c, s, st, y.size), y)
        y, c, s = oracle.mxfp4(t)
        assert np.array_equal(oracle.mxfp4_decode(c, s, y.size), y)
        y, b = oracle.q4k(t)
        assert np.array_equal(oracle.q4k_decode(b, y.size), y)


# ----------------------------------------------------------------------------- idempotence / monotonicity
def test_mxfp4_is_idempotent():
    x = rand_bf16(64, 512, 5)
    y, c, s = oracle.mxfp4(x)
    y2, c2, s2 = oracle.mxfp4(y.reshape(64, 512))
    assert np.array_equal(y, y2) and np.array_equal(c, c2) and np.array_equal(s, s2)


def test_nvfp4_monotone_within_block():
    rng = np.random.default_rng(1)
    v = np.sort(rng.standard_normal(4096).astype(np.float32) * 0.02)
    xb = ((v.view(np.uint32) + 0x8000) >> 16).astype(np.uint16)    # any BF16 values, sorted
    xb = np.sort(f32_of(xb)).astype(np.float32).view(np.uint32) >> 16
    xb = xb.astype(np.uint16).reshape(256, 16)
    # one shared block scale: give every block the same max by construction
    xb[:, -1] = bits_of(np.float32([0.125]))[0]
    for row in xb:
        y, _, _, _ = oracle.nvfp4(row.reshape(1, 16), 0.125)
        yf = f32_of(y)
        assert np.all(np.diff(yf) >= 0)


# ----------------------------------------------------------------------------- degenerate cases
def test_mxfp4_blocks_below_2_pow_minus_124_take_byte_0():
    """A block whose max is below 2^-124 has floor(log2 amax) - 2 < -127, so its E8M0 byte
    clamps to 0 (e = -127).  Its codes are the nearest E2M1 values of x * 2^127, and y is
    code * 2^-127 exactly: float64 arithmetic here, nonzero codes included."""
    rng = np.random.default_rng(31)
    h = rng.integers(0x0080, 0x00C0, (4, 256)).astype(np.uint16)      # 2^-126 .. 1.5 * 2^-126
    h |= (rng.random((4, 256)) < 0.5).astype(np.uint16) << 15
    h[1, 32:64] = rng.integers(0x0001, 0x0080, 32).astype(np.uint16)  # BF16 subnormals
    y, c, s = oracle.mxfp4(h)
    assert np.all(s == 0)
    xf = f32_of(h).astype(np.float64).reshape(-1)
    a = np.abs(xf * 2.0 ** 127)
    dist = np.abs(a[:, None] - E2M1[None, :])
    cand = dist == dist.min(axis=1, keepdims=True)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    got = unpack_nibbles(c)
    assert np.array_equal(got & 7, idx)
    assert np.count_nonzero(got & 7) > 100
    want = bits_of((e2m1_val(got) * 2.0 ** -127).astype(np.float32))
    # a value that rounds to code 0 keeps its sign: -0 for negative inputs
    want = np.where((got & 7) == 0, (h.reshape(-1) & 0x8000), want).astype(np.uint16)
    assert np.array_equal(y, want)


def test_degenerate_inputs():
    z = np.zeros((2, 64), np.uint16)
    z[0, 3] = 0x8000                                            # a negative zero
    y, c, s, st = oracle.nvfp4(z, 0.0)
    assert st == 0.0 and np.all(s == 0)
    assert unpack_nibbles(c)[3] == 8 and np.all(np.delete(unpack_nibbles(c), 3) == 0)
    assert np.array_equal(y, z.reshape(-1))
    y, c, s = oracle.mxfp4(z)
    assert np.all(s == 0) and np.array_equal(y, z.reshape(-1))
    y, b = oracle.q4k(np.zeros((1, 256), np.uint16))
    assert np.all(y == 0) and np.all(b == 0)
    # a tensor of BF16 subnormals: scales underflow, no NaN anywhere
    tiny = np.full((1, 32), 0x0001, np.uint16)
    tiny[0, ::2] = 0x8003
    y, c, s, st = oracle.nvfp4(tiny, oracle.amax(tiny))
    assert not np.any(np.isnan(f32_of(y)))
    y, c, s = oracle.mxfp4(tiny)
    assert np.all(s == 0) and not np.any(np.isnan(f32_of(y)))


def test_nvfp4_block_whose_scale_underflows_encodes_signed_zeros():
    """A block far below the tie-group max gets E4M3 scale 0 (amax_b / (6 s_t) rounds to
    0), so S = 0 and inv = 0: every element encodes as a zero of its own sign (code 0 or
    8) and dequantizes to that zero, whatever its magnitude."""
    x = np.zeros((1, 64), np.float32)
    x[0, 0] = 1.0                                   # the group max: s_t = 1 / 2688
    rng = np.random.default_rng(41)
    x[0, 16:] = rng.uniform(1e-9, 2e-9, 48) * np.where(rng.random(48) < 0.5, -1.0, 1.0)
    h = bits_of(torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy())
    y, c, s, st = oracle.nvfp4(h, 1.0)
    assert st == np.float32(1.0) / np.float32(2688.0)
    assert s[0] != 0 and np.all(s[1:] == 0)
    got = unpack_nibbles(c)[16:]
    sign = (h[0, 16:] >> 15).astype(np.uint8)
    assert np.all(got == 8 * sign)                  # +0 for positive inputs, -0 for negative
    assert np.array_equal(y.reshape(-1)[16:], (h[0, 16:] & 0x8000).astype(np.uint16))


def test_nvfp4_scale_reciprocal_overflow_keeps_zero_signs():
    """A block scale S below 2^-128 has 1/S = inf; zeros stay zeros of their sign."""
    x = np.zeros((1, 16), np.uint16)
    x[0, 0] = 0x0001                                           # 2^-133
    x[0, 1] = 0x8000
    y, c, s, st = oracle.nvfp4(x, oracle.amax(x))
    cc = unpack_nibbles(c)
    assert cc[1] == 8 and np.all(cc[2:] == 0)
    assert not np.any(np.isnan(f32_of(y)))


# ----------------------------------------------------------------------------- STE
def test_ste_identity_is_a_bitwise_copy():
    g = workloads.normal_with_outliers(8, 256, 1e-3, 0, 1, 3, 9)
    gb = workloads.bf16_bits(g).reshape(-1)
    assert np.array_equal(oracle.ste_backward(g), gb)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_ste_clipped_mask_is_saturation(fmt):
    x = rand_bf16(8, 512, 17)
    g = workloads.normal_with_outliers(8, 512, 1e-3, 0, 1, 3, 10)
    gb = workloads.bf16_bits(g).reshape(-1)
    xf = f32_of(workloads.bf16_bits(x).reshape(-1))
    am = oracle.amax(x)
    gx = oracle.ste_backward(g, 1, fmt, x, am)
    if fmt == "nvfp4":
        _, _, s, st = oracle.nvfp4(x, am)
        S = (s.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(st)).astype(np.float32)
        inv = np.where(S == 0, 0, np.float32(1) / S).astype(np.float32)
        q = (xf.reshape(-1, 16) * inv[:, None]).astype(np.float32).reshape(-1)
        keep = np.abs(q) <= 6
    elif fmt == "mxfp4":
        _, _, s = oracle.mxfp4(x)
        q = xf.reshape(-1, 32).astype(np.float64) * np.exp2(127.0 - s.astype(np.float64))[:, None]
        keep = np.abs(q.reshape(-1)) <= 6
    else:
        keep = np.ones(xf.size, bool)
        for sbi in range(xf.size // 256):
            d, dm, sc, m, _ = oracle.q4k_fit_one(workloads.bf16_bits(x).reshape(-1)[256 * sbi:256 * sbi + 256])
            d = np.float32(np.uint16(d).view(np.float16))
            dm = np.float32(np.uint16(dm).view(np.float16))
            for j in range(8):
                s_ = np.float32(d * np.float32(sc[j]))
                mm = np.float32(dm * np.float32(m[j]))
                inv = np.float32(0) if s_ == 0 else np.float32(1) / s_
                k = slice(256 * sbi + 32 * j, 256 * sbi + 32 * j + 32)
                v = ((xf[k] + mm).astype(np.float32) * inv).astype(np.float32)
                keep[k] = (v >= 0) & (v <= 15)
    assert np.array_equal(gx, np.where(keep, gb, 0).astype(np.uint16))
    if fmt == "nvfp4":
        assert (~keep).sum() > 0                               # saturation does occur


def test_q4k_clipped_ste_keeps_both_ends_of_the_code_range():
    """The Q4_K clipped STE keeps the gradient where 0 <= (x + mm) * inv <= 15, ends
    included.  The super-block of workloads.q4k_ste_ends hits both ends exactly (its
    construction is checked here: d = 2^-8, dmin = 65 * 2^-20, sc[1] = 32, m[2] = 1), and
    its element at -2^-8 lies below its quantized offset and is clipped."""
    xb = workloads.q4k_ste_ends()
    h = workloads.bf16_bits(xb).reshape(1, 256)
    d, dm, sc, m, q = oracle.q4k_fit_one(h)
    f16 = np.array([d, dm], np.uint16).view(np.float16).astype(np.float64)
    assert f16[0] == 2.0 ** -8 and f16[1] == 65 * 2.0 ** -20
    assert sc[1] == 32 and m[2] == 1 and m[1] == 0 and q[32] == 15 and q[64] == 0
    g = torch.ones(1, 256, dtype=torch.bfloat16)
    gx = oracle.ste_backward(g, 1, "q4k", xb).reshape(-1)
    one = workloads.bf16_bits(g).reshape(-1)[0]
    assert gx[32] == one                             # (x + mm) * inv == 15 exactly
    assert gx[64] == one                             # (x + mm) * inv == 0 exactly
    assert gx[1] == 0                                # (x + mm) * inv < 0: clipped


def test_q4k_negative_values_rounding_to_code_zero_dequantize_to_positive_zero():
    """Q4_K codes are unsigned integers: a sub-block whose stored min is 0 but that
    holds small negative values dequantizes them from the integer code 0 to +0."""
    x = np.zeros(256, np.float32)
    x[:32] = np.linspace(0, 1, 32, dtype=np.float32)
    x[5] = -1e-4                                              # rounds to q = 0
    x[32:64] = -1.0                                           # a large min elsewhere: dmin = 1/63,
                                                              # so the first sub-block's m is 0
    xb = oracle.f32_to_bf16(x)
    d, dm, sc, m, q = oracle.q4k_fit_one(xb)
    assert m[0] == 0 and q[5] == 0
    y, _ = oracle.q4k(xb.reshape(1, 256))
    assert y[5] == 0x0000


# ----------------------------------------------------------------------------- FP32 latent input
def test_f32_input_equal_to_bf16_path_when_representable():
    """FP32 master weights that happen to be BF16 values quantize exactly like the BF16 tensor."""
    x = rand_bf16(16, 512, 31)
    xf = x.float()
    am = oracle.amax(x)
    assert oracle.amax(xf) == am
    for a, b in zip(oracle.nvfp4(x, am), oracle.nvfp4(xf, am)):
        assert np.array_equal(a, b)
    for a, b in zip(oracle.mxfp4(x), oracle.mxfp4(xf)):
        assert np.array_equal(a, b)
    for a, b in zip(oracle.q4k(x), oracle.q4k(xf)):
        assert np.array_equal(a, b)


def test_f32_nvfp4_on_grid_codes_round_trip():
    """x = code * sb * s_t with an 18-bit s_t: exact in FP32 but not in BF16; the fit
    recovers every code and block scale, and y = BF16(x)."""
    rng = np.random.default_rng(41)
    rows, cols = 8, 256
    nb = rows * cols // 16
    st = np.float32((1.0 + rng.integers(1, 1 << 17) / 2.0 ** 17) * 2.0 ** -10)
    sb = rng.integers(0x08, 0x7F, size=nb).astype(np.uint8)
    sb[3] = 0x7E
    sbv = sb.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    codes = rng.integers(0, 16, size=(nb, 16)).astype(np.uint8)
    codes[np.arange(nb), rng.integers(0, 16, nb)] = 7
    x64 = e2m1_val(codes) * sbv[:, None] * float(st)
    x = x64.astype(np.float32)
    assert np.array_equal(x.astype(np.float64), x64)                # exact in FP32
    x = x.reshape(rows, cols)
    am = oracle.amax(x)
    y, c, s, st_out = oracle.nvfp4(x, am)
    assert st_out == st
    assert np.array_equal(s, sb) and np.array_equal(unpack_nibbles(c), codes.reshape(-1))
    assert np.array_equal(y, oracle.f32_to_bf16(x.reshape(-1)))


def test_f32_codes_brute_force_and_decoder():
    rng = np.random.default_rng(43)
    x = (rng.standard_normal((8, 512)) * 0.02).astype(np.float32)
    x[2, 5] = 0.7                                                    # an outlier
    xf = x.reshape(-1)
    am = oracle.amax(x)
    # NVFP4: nearest E2M1 of x * (1/S) with S from the block scale, ties to even
    y, c, s, st = oracle.nvfp4(x, am)
    S = (s.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(st)).astype(np.float32)
    inv = np.where(S == 0, np.float32(0), np.float32(1) / S).astype(np.float32)
    q = (xf.reshape(-1, 16) * inv[:, None]).astype(np.float32).reshape(-1)
    lib = q.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(e2m1_val(unpack_nibbles(c)).astype(np.float32), np.abs(lib) *
                          np.where(q.view(np.uint32) >> 31, -1, 1))
    assert np.array_equal(oracle.nvfp4_decode(c, s, st, xf.size), y)
    # MXFP4 and Q4_K: the independent decoder reproduces the dequantized output
    y, c, s = oracle.mxfp4(x)
    assert np.array_equal(oracle.mxfp4_decode(c, s, xf.size), y)
    e = s.astype(np.int64) - 127
    qm = (xf.reshape(-1, 32).astype(np.float64) * np.exp2(-e.astype(np.float64))[:, None])
    assert np.array_equal(e2m1_val(unpack_nibbles(c)).astype(np.float64),
                          qm.reshape(-1).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
                          .astype(np.float64))
    y, b = oracle.q4k(x)
    assert np.array_equal(oracle.q4k_decode(b, xf.size), y)


def test_codes_and_scales_stay_in_range():
    """Every stored field is a valid value of its type, even for extreme inputs.
    E4M3 scales are finite and at most 448 (never the NaN encodings 0x7F / 0xFF) and
    never negative. E8M0 bytes are never 0xFF (NaN). Q4_K d and dmin are finite,
    non-negative FP16, and sc, m fit 6 bits."""
    rng = np.random.default_rng(11)
    mags = [1e-30, 1e-6, 0.02, 1.0, 3e4, 3e38]
    xs = []
    for m in mags:
        a = rng.standard_normal((4, 256)).astype(np.float32) * np.float32(m)
        a[0, :7] = [0.0, -0.0, m, -m, 6 * m, -448 * m, 1e-45]
        xs.append(workloads.to_bf16(a))
    for x in xs:
        xb = workloads.bf16_bits(x)
        f = np.abs(x.float().numpy())
        if np.isfinite(f).all() and f.max() < 1e38:
            _, _, sc, _ = oracle.nvfp4(xb, float(f.max()))
            assert not np.any((sc & 0x7F) == 0x7F) and not np.any(sc & 0x80)
            assert np.all(sc.view(ml_dtypes.float8_e4m3fn).astype(np.float32) <= 448.0)
        _, _, e8 = oracle.mxfp4(xb)
        assert not np.any(e8 == 0xFF)
        if f.max() < 4e6:                      # inside the Q4_K range: 63 * 65504 bounds min_j
            _, blocks = oracle.q4k(xb)
            blk = blocks.reshape(-1, 144)
            d = blk[:, 0:2].copy().view(np.float16).astype(np.float32)
            dm = blk[:, 2:4].copy().view(np.float16).astype(np.float32)
            assert np.isfinite(d).all() and np.isfinite(dm).all()
            assert (d >= 0).all() and (dm >= 0).all()
