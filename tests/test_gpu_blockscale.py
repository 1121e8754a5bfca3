"""The NVFP4 block scale from a tie group's tables (nv_block_scale_tab: the ratio by
a reciprocal taken once per group, S and 1/S by lookup) against the plain derivation
with one IEEE division and one reciprocal per block (nv_block_scale), bit for bit in
the block byte, S and 1/S.

Every non-negative BF16 block amax (+inf and the NaN patterns included) and 2^18
pseudo-random non-negative FP32 ones are tried under several hundred tensor scales:
s_t = amax_g / 2688 for log-uniform amax_g over 2^-126..2^126, for typical weight
maxima, powers of two, and the edges of the range where the table path applies
(6 s_t in [2^-80, 2^100]; outside it every block takes the division).  The plain
derivation is the one the oracle's parity tests already pin, so agreement here carries
that parity over to the kernels that use the tables."""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe():
    spec = importlib.util.spec_from_file_location("build_probe",
                                                  os.path.join(HERE, "cuda", "build_probe.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = ctypes.CDLL(mod.build())
    P = ctypes.c_void_p
    lib.probe_blockscale.argtypes = [P, ctypes.c_int, ctypes.c_uint32, P, P, P]
    lib.probe_blockscale.restype = ctypes.c_int
    return lib


def tensor_scales():
    rng = np.random.default_rng(2688)
    f = np.float32
    amax = [f(2.0) ** rng.uniform(-126, 126, 240).astype(np.float32),
            rng.uniform(0.01, 100.0, 120).astype(np.float32),
            f(2.0) ** np.arange(-120, 121, 8, dtype=np.float32),
            np.float32([0.0, 1.0, 448.0, 2688.0, 3.3895314e38, 1e-45])]
    st = [np.concatenate(amax).astype(np.float32) / f(2688.0)]
    # 6 s_t at and around the ends of the table range
    for edge in (f(2.0) ** -80, f(2.0) ** 100):
        base = edge / f(6.0)
        bits = base.view(np.uint32) + np.arange(-3, 4, dtype=np.int64).astype(np.uint32)
        st.append(bits.view(np.float32))
    return np.concatenate(st).astype(np.float32)


def test_table_block_scale_equals_division(probe):
    st = tensor_scales()
    d_st = torch.from_numpy(st).cuda()
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(16, dtype=torch.int32, device="cuda")
    fast = torch.zeros(len(st), dtype=torch.int64, device="cuda")
    n_f32 = 1 << 18
    assert probe.probe_blockscale(d_st.data_ptr(), len(st), n_f32, bad.data_ptr(),
                                  first.data_ptr(), fast.data_ptr()) == 0
    nbad = int(bad.item())
    rec = first.cpu().numpy().view(np.uint32).reshape(4, 4)[:min(nbad, 4)]
    assert nbad == 0, [(float(st[r[0]]), hex(r[1]), int(r[2]), int(r[3])) for r in rec]
    # the table path decides nearly every block itself where it applies
    total = 32768 + n_f32
    six = (np.float32(6.0) * st).astype(np.float32)
    inside = (six >= np.float32(2.0) ** -80) & (six <= np.float32(2.0) ** 100)
    frac = fast.cpu().numpy() / total
    assert inside.sum() > 300
    assert np.all(frac[~inside] == 0)
    assert np.median(frac[inside]) > 0.95, np.median(frac[inside])
