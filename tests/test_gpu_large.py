"""More than 2^31 elements in one tensor: every index in the kernels is 64-bit.

A [32769, 65536] BF16 tensor holds 2,147,549,184 elements (4.3 GB).  Its last row
starts at element 2^31, so a 32-bit element index or byte offset anywhere in a
kernel would wrap there.  The oracle checks sampled rows on both sides of that point.
The NVFP4 tensor amax is checked against torch's own reduction of |x| on the device
(max is exact)."""
import pytest
import torch

import fp4_fake_quant_b200 as qf
from gpu_helpers import DEV, bits, compare_rows, u8

pytestmark = pytest.mark.gpu

ROWS, COLS = 32769, 65536
SAMPLE = [0, 1, 16384, 32767, 32768]


@pytest.fixture(scope="module")
def big():
    free, _ = torch.cuda.mem_get_info()
    if free < 14 * (1 << 30):
        pytest.skip("needs ~14 GB of free device memory")
    g = torch.Generator(device=DEV).manual_seed(2024)
    x = (torch.randn(ROWS, COLS, generator=g, device=DEV, dtype=torch.float32) * 0.02).to(
        torch.bfloat16)
    x[ROWS - 1, COLS - 5] = 3.0                      # the tensor amax sits past element 2^31
    yield x
    del x
    torch.cuda.empty_cache()


def _rows_cpu(x, rows):
    return {r: x[r:r + 1].cpu() for r in rows}


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "q4k"])
def test_beyond_2_31_elements(big, fmt):
    assert big.numel() > 2 ** 31
    y, c, s = qf.alloc_outputs(fmt, big)
    kw = {}
    am = 0.0
    if fmt == "nvfp4":
        amax = torch.empty(1, device=DEV)
        qf.qf_amax_tied([big], [0], amax)
        ref = big.abs().max().float()
        torch.cuda.synchronize()
        assert amax.item() == ref.item() == 3.0
        kw = {"groups": [0], "group_amax": amax}
        am = float(amax.item())
    qf.qf_fakequant(fmt, [big], [y], [c], [s] if s is not None else None, **kw)
    torch.cuda.synchronize()
    q4 = fmt == "q4k"
    cpr = COLS // 2 if not q4 else COLS // 256 * 144
    spr = 0 if q4 else COLS // (16 if fmt == "nvfp4" else 32)
    xs = _rows_cpu(big, SAMPLE)
    for r in SAMPLE:
        yb = bits(y[r:r + 1])
        cb = u8(c[r * cpr:(r + 1) * cpr])
        sb = u8(s[r * spr:(r + 1) * spr]) if spr else None
        compare_rows(fmt, xs[r], yb, cb, sb, [0], am, label=f"{fmt} row {r}")
    del y, c, s
    torch.cuda.empty_cache()
