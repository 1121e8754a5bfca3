"""Division by the Q4_K fits' constant divisors (div_const: a product with the rounded
reciprocal and one correction by the exact residual) against the IEEE division
__fdiv_rn, on EVERY binary32 input, for each constant the kernels divide by: 15 and 63
(the min/max fit: the sub-block scale, the super-block d and dmin) and the MSE search's
trial divisors 14, 14.5, 15.5, 16, 16.5, 17, 17.5, 18.  The reciprocal is passed as the
kernels compute it, RN(1/c) in binary32."""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DIVISORS = [15.0, 63.0, 14.0, 14.5, 15.5, 16.0, 16.5, 17.0, 17.5, 18.0]


@pytest.fixture(scope="module")
def probe():
    spec = importlib.util.spec_from_file_location("build_probe",
                                                  os.path.join(HERE, "cuda", "build_probe.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = ctypes.CDLL(mod.build())
    lib.probe_divconst.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_uint32,
                                   ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    lib.probe_divconst.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("c", DIVISORS)
def test_div_const_equals_division_on_every_input(probe, c):
    c_inv = float(np.float32(1.0) / np.float32(c))
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert probe.probe_divconst(c, c_inv, 0, 1 << 32, bad.data_ptr(), first.data_ptr()) == 0
    n = int(bad.item())
    assert n == 0, (c, n, hex(int(first.item()) & 0xFFFFFFFF))
