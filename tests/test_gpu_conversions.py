"""The hardware conversions the kernels use, against the oracle, on EVERY binary32
input (both signs, subnormals included, NaN patterns excluded).

A probe runs the library's own device helpers (cvt.rn.satfinite.e2m1x2.f32,
cvt.rn.satfinite.e4m3x2.f32, cvt.rn.bf16x2.f32, __float2half_rn) over every bit
pattern of a sign and records each pattern where the result changes.  Within one
sign the patterns are ordered by magnitude and both sides are monotone step
functions (the oracle's monotonicity is pinned by a CPU test), so agreeing at
every change point and at the pattern just before it means agreeing everywhere.
"""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
RANGES = {"pos": (0x00000000, 0x7F7FFFFF), "neg": (0x80000000, 0xFF7FFFFF)}
NAMES = {0: "e2m1", 1: "e4m3", 2: "bf16", 3: "f16"}
ORACLE = {0: oracle.e2m1_from_f32, 1: oracle.e4m3_from_f32, 2: oracle.f32_to_bf16,
          3: oracle.f32_to_f16}


@pytest.fixture(scope="module")
def probe():
    spec = importlib.util.spec_from_file_location("build_probe",
                                                  os.path.join(HERE, "cuda", "build_probe.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = ctypes.CDLL(mod.build())
    P, U32 = ctypes.c_void_p, ctypes.c_uint32
    lib.probe_scan.argtypes = [ctypes.c_int, U32, U32, P, P, U32, P]
    lib.probe_pairs.argtypes = [P, P, ctypes.c_int, P, P, P]
    lib.probe_decode.argtypes = [P, P]
    for f in (lib.probe_scan, lib.probe_pairs, lib.probe_decode):
        f.restype = ctypes.c_int
    return lib


def scan(lib, which, lo, hi, cap=1 << 20):
    pos = torch.zeros(cap, dtype=torch.int32, device="cuda")
    val = torch.zeros(cap, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert lib.probe_scan(which, lo, hi, pos.data_ptr(), val.data_ptr(), cap, count.data_ptr()) == 0
    n = int(count.item())
    assert 0 < n <= cap
    p = pos[:n].cpu().numpy().view(np.uint32)
    v = val[:n].cpu().numpy().view(np.uint32)
    order = np.argsort(p)
    return p[order], v[order]


@pytest.mark.parametrize("sign", ["pos", "neg"])
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_conversion_equals_oracle_on_every_pattern(probe, which, sign):
    lo, hi = RANGES[sign]
    p, v = scan(probe, which, lo, hi)
    assert p[0] == lo
    conv = ORACLE[which]
    at = conv(p.view(np.float32)).astype(np.uint32)
    assert np.array_equal(at, v), f"{NAMES[which]}: differs at a change point"
    before = conv((p[1:] - 1).view(np.float32)).astype(np.uint32)
    assert np.array_equal(before, v[:-1]), f"{NAMES[which]}: differs just before a change point"
    assert int(conv(np.array([hi], np.uint32).view(np.float32))[0]) == int(v[-1])


def test_packed_pair_layout(probe):
    rng = np.random.default_rng(4)
    a = (rng.standard_normal(4096) * 3).astype(np.float32)
    b = (rng.standard_normal(4096) * 3).astype(np.float32)
    da, db = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    outs = [torch.zeros(4096, dtype=torch.int32, device="cuda") for _ in range(3)]
    assert probe.probe_pairs(da.data_ptr(), db.data_ptr(), 4096, *[o.data_ptr() for o in outs]) == 0
    e2m1, e4m3, bf16 = [o.cpu().numpy().view(np.uint32) for o in outs]
    ua, ub = oracle.e2m1_from_f32(a).astype(np.uint32), oracle.e2m1_from_f32(b).astype(np.uint32)
    assert np.array_equal(e2m1, (ua << 4) | ub)              # first operand -> high nibble
    ua, ub = oracle.e4m3_from_f32(a).astype(np.uint32), oracle.e4m3_from_f32(b).astype(np.uint32)
    assert np.array_equal(e4m3, (ua << 8) | ub)
    ua, ub = oracle.f32_to_bf16(a).astype(np.uint32), oracle.f32_to_bf16(b).astype(np.uint32)
    assert np.array_equal(bf16, (ua << 16) | ub)


def test_decode_conversions(probe):
    o1 = torch.zeros(256, dtype=torch.int32, device="cuda")
    o2 = torch.zeros(256, dtype=torch.int32, device="cuda")
    assert probe.probe_decode(o1.data_ptr(), o2.data_ptr()) == 0
    e2m1 = o1.cpu().numpy().view(np.uint32)
    e4m3 = o2.cpu().numpy().view(np.uint32)
    for byte in range(256):
        lo = np.float16(oracle.e2m1_to_f32(byte & 15)).view(np.uint16)
        hi = np.float16(oracle.e2m1_to_f32(byte >> 4)).view(np.uint16)
        assert e2m1[byte] == (int(hi) << 16) | int(lo), byte
        want = np.float16(oracle.e4m3_to_f32(byte))
        got = np.uint16(e4m3[byte] & 0xFFFF).view(np.float16)
        assert (np.isnan(want) and np.isnan(got)) or want.view(np.uint16) == got.view(np.uint16)
