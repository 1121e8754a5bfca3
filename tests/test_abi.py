"""The C ABI boundary on the host (no GPU needed): libqf.so loads, exports every
entry point include/qf.h declares, and rejects invalid calls with the documented
status codes before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qf.h")


@pytest.fixture(scope="module")
def qf():
    from fp4_fake_quant_b200 import _build
    _build.build()
    import fp4_fake_quant_b200 as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qf_[a-z_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("qf_amax_tied", "qf_fakequant", "qf_pack", "qf_ste_backward"):
        assert n in names


def test_library_exports_every_declared_symbol(qf):
    out = subprocess.run(["nm", "-D", "--defined-only", qf.binding.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (qf_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(qf.lib, n)
    assert set(qf.EXPORTS) == set(declared_functions())


def test_header_compiles_as_c():
    src = '#include "qf.h"\nint main(void){ qf_tensor t = {0}; (void)t; return (int)QF_OK; }\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                        "-x", "c", "-", "-fsyntax-only"], input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls(qf, tmp_path):
    """The boundary is usable from plain C: a C99 program links libqf.so and gets the
    documented answers from calls that need no GPU."""
    src = r"""
#include <stdio.h>
#include <string.h>
#include "qf.h"
int main(void) {
    qf_tensor t;
    memset(&t, 0, sizeof t);
    t.x = (const void*)0x1000; t.rows = 4; t.cols = 48; t.y = (void*)0x2000;
    t.codes = (void*)0x3000; t.scales = (void*)0x4000;
    if (qf_version() != ((1 << 16) | 7)) return 1;
    if (strncmp(qf_status_string(QF_ERR_SHAPE), "QF_ERR_SHAPE", 12) != 0) return 2;
    if (qf_fakequant(QF_MXFP4, &t, 1, NULL, 0, NULL, NULL) != QF_ERR_SHAPE) return 3;
    if (qf_last_error()[0] == 0) return 4;
    if (qf_amax_fakequant_workspace_bytes(1) != 256) return 5;
    if (qf_amax_tied(&t, 1, NULL, 1, NULL, NULL) != QF_ERR_INVALID_ARG) return 6;
    printf("ok\n");
    return 0;
}
"""
    c = tmp_path / "abi.c"
    c.write_text(src)
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(qf.binding.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                        str(c), "-L", lib_dir, "-lqf", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_struct_layout_matches_header(qf):
    T = qf.binding.QfTensor
    assert ctypes.sizeof(T) == 56
    assert T.y.offset == 32 and T.codes.offset == 40 and T.scales.offset == 48


def test_status_strings(qf):
    for s in range(7):
        assert qf.lib.qf_status_string(s).decode().startswith("QF_")
    assert qf.lib.qf_version() == (1 << 16) | 7


def _tensor(qf, x=0x1000, rows=4, cols=64, group=0, y=0x2000, codes=0x3000, scales=0x4000,
            x_type=0):
    arr = (qf.binding.QfTensor * 1)()
    t = arr[0]
    t.x, t.rows, t.cols, t.group, t.x_type = x, rows, cols, group, x_type
    t.y, t.codes, t.scales = y, codes, scales
    return arr


def _fq(qf, f, arr, n=1, amax=None, ng=0, pack=False):
    fn = qf.lib.qf_pack if pack else qf.lib.qf_fakequant
    return fn(f, arr, n, amax, ng, None, None)


@pytest.mark.parametrize("pack", [False, True])
def test_validation_codes(qf, pack):
    OK, INV, SHAPE, ALIGN, UNSUP = 0, 1, 2, 3, 4
    assert _fq(qf, 7, _tensor(qf), pack=pack) == UNSUP
    assert _fq(qf, 1, _tensor(qf), n=-1, pack=pack) == INV
    assert _fq(qf, 1, None, n=1, pack=pack) == INV
    assert _fq(qf, 1, _tensor(qf), n=0, pack=pack) == OK              # nothing to do
    assert _fq(qf, 1, _tensor(qf, cols=48), pack=pack) == SHAPE        # 48 % 32
    assert _fq(qf, 2, _tensor(qf, cols=512 + 32), pack=pack) == SHAPE  # Q4_K needs 256
    assert _fq(qf, 0, _tensor(qf, cols=24), amax=0x5000, ng=1, pack=pack) == SHAPE
    assert _fq(qf, 1, _tensor(qf, rows=-1), pack=pack) == SHAPE
    assert _fq(qf, 1, _tensor(qf, rows=1 << 40, cols=1 << 30), pack=pack) == SHAPE
    assert _fq(qf, 1, _tensor(qf, x=0x1008), pack=pack) == ALIGN
    assert _fq(qf, 1, _tensor(qf, codes=0x3004), pack=pack) == ALIGN
    assert _fq(qf, 1, _tensor(qf, x=0), pack=pack) == INV
    assert _fq(qf, 1, _tensor(qf, x_type=2), pack=pack) == UNSUP
    two = (qf.binding.QfTensor * 2)(_tensor(qf)[0], _tensor(qf, x_type=1)[0])
    assert _fq(qf, 1, two, n=2, pack=pack) == INV                    # mixed element types
    assert _fq(qf, 1, _tensor(qf, y=0, codes=0, scales=0), pack=pack) == INV
    # Q4_K ignores `scales`: a pack with no codes has no output
    assert _fq(qf, 2, _tensor(qf, cols=256, codes=0), pack=True) == INV
    # NVFP4 needs the group amax and a valid group
    assert _fq(qf, 0, _tensor(qf), amax=None, ng=1, pack=pack) == INV
    assert _fq(qf, 0, _tensor(qf), amax=0x5000, ng=0, pack=pack) == INV
    assert _fq(qf, 0, _tensor(qf, group=1), amax=0x5000, ng=1, pack=pack) == INV
    assert _fq(qf, 0, _tensor(qf, group=-1), amax=0x5000, ng=1, pack=pack) == INV
    # a tensor's input and outputs must be disjoint
    if not pack:                                   # (qf_pack ignores y)
        assert _fq(qf, 1, _tensor(qf, y=0x1100), pack=pack) == INV
    assert _fq(qf, 1, _tensor(qf, codes=0x1100), pack=pack) == INV
    assert _fq(qf, 1, _tensor(qf, scales=0x3010), pack=pack) == INV        # inside codes
    assert _fq(qf, 2, _tensor(qf, cols=256, codes=0x10F0), pack=pack) == INV  # Q4_K blocks over x
    # empty tensors are skipped without needing outputs
    assert _fq(qf, 1, _tensor(qf, rows=0, y=0, codes=0, scales=0), pack=pack) == OK
    assert qf.lib.qf_last_error() == b""


def test_valid_call_without_a_gpu_reports_cuda_error(qf):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fq(qf, 1, _tensor(qf)) == 5
    assert qf.lib.qf_last_error().decode()


def test_adjacent_buffers_are_disjoint(qf):
    """Buffers that touch but do not overlap pass validation: x, y, codes and scales
    laid out back to back (4 x 64 MXFP4: 512 B of x, 512 B of y, 128 B of codes, 8 B of
    scales).  Without a GPU the call then fails at its first CUDA step (QF_ERR_CUDA),
    which shows that the argument checks accepted it."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present (the pointers are fake)")
    arr = _tensor(qf, x=0x10000, y=0x10200, codes=0x10400, scales=0x10480)
    assert _fq(qf, 1, arr) == 5
    assert "overlap" not in qf.lib.qf_last_error().decode()
    arr = _tensor(qf, x=0x10000, y=0x101F0)        # y starts 16 bytes before x ends
    assert _fq(qf, 1, arr) == 1


def test_amax_and_ste_validation(qf):
    INV, SHAPE, ALIGN, UNSUP = 1, 2, 3, 4
    lib = qf.lib
    arr = _tensor(qf, cols=7)                       # any cols is fine for the amax
    assert lib.qf_amax_tied(arr, 1, None, 1, None, None) == INV
    assert lib.qf_amax_tied(arr, 1, 0x5000, 0, None, None) == INV
    assert lib.qf_amax_tied(_tensor(qf, group=2), 1, 0x5000, 2, None, None) == INV
    assert lib.qf_amax_tied(_tensor(qf, x=0x1002), 1, 0x5000, 1, None, None) == ALIGN
    assert lib.qf_amax_tied(None, 1, 0x5000, 1, None, None) == INV
    assert lib.qf_ste_backward(0, 0x1000, 0x2000, 64, 2, None, None, 0, None) == UNSUP
    assert lib.qf_ste_backward(0, 0x1000, 0x2000, -1, 0, None, None, 0, None) == SHAPE
    assert lib.qf_ste_backward(0, 0x1008, 0x2000, 64, 0, None, None, 0, None) == ALIGN
    assert lib.qf_ste_backward(0, 0, 0x2000, 64, 0, None, None, 0, None) == INV
    assert lib.qf_ste_backward(0, 0x1000, 0x1000, 64, 0, None, None, 0, None) == 0  # aliased
    assert lib.qf_ste_backward(0, 0x1000, 0x1010, 64, 0, None, None, 0, None) == INV  # partly
    assert lib.qf_ste_backward(9, 0x1000, 0x2000, 256, 1, _tensor(qf), None, 0, None) == UNSUP
    assert lib.qf_ste_backward(1, 0x1000, 0x2000, 256, 1, None, None, 0, None) == INV
    assert lib.qf_ste_backward(1, 0x1000, 0x2000, 255, 1, _tensor(qf), None, 0, None) == SHAPE
    assert lib.qf_ste_backward(0, 0x1000, 0x2000, 256, 1, _tensor(qf), None, 1, None) == INV


def test_amax_fakequant_validation(qf):
    """qf_amax_fakequant makes every check of qf_amax_tied and qf_fakequant(NVFP4),
    plus its workspace checks, before anything launches."""
    INV, SHAPE, ALIGN = 1, 2, 3
    lib = qf.lib
    wb = lib.qf_amax_fakequant_workspace_bytes
    assert wb(0) == 0 and wb(-3) == 0
    assert wb(1) == 256 and wb(60) == 256 and wb(61) == 512      # 4 header words + 1 per group
    assert qf.workspace_bytes(256) == 1280

    def call(arr, n=1, amax=0x5000, ng=1, ws=0x9000, wsb=256):
        return lib.qf_amax_fakequant(arr, n, amax, ng, None, None, ws, wsb, None)

    assert call(_tensor(qf), n=-1) == INV
    assert call(None) == INV
    assert call(_tensor(qf), ng=0) == INV
    assert call(_tensor(qf), amax=None) == INV
    assert call(_tensor(qf), wsb=255) == INV                       # workspace too small
    assert call(_tensor(qf), ng=61, wsb=256) == INV
    assert call(_tensor(qf), ws=0x9008) == ALIGN
    assert call(_tensor(qf, cols=24)) == SHAPE                     # NVFP4 needs 16 | cols
    assert call(_tensor(qf, group=1)) == INV
    assert call(_tensor(qf, y=0, codes=0, scales=0)) == INV
    assert call(_tensor(qf, codes=0x3004)) == ALIGN
    assert call(_tensor(qf, x=0x1008)) == ALIGN
    two = (qf.binding.QfTensor * 2)(_tensor(qf)[0], _tensor(qf, x_type=1)[0])
    assert call(two, n=2) == INV
    assert call(_tensor(qf, y=0x1100)) == INV                      # y overlaps x
    assert lib.qf_workspace_check(None, None) == INV


def test_product_path_has_no_oracle_dependency():
    """The library and its binding never import, link or read the oracle."""
    pkg = os.path.join(ROOT, "fp4_fake_quant_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f
    out = subprocess.run(["ldd", os.path.join(pkg, "libqf.so")], capture_output=True,
                         text=True).stdout
    assert "oracle" not in out


def test_lora_validation(qf):
    INV, SHAPE, ALIGN, UNSUP = 1, 2, 3, 4
    lib = qf.lib
    L = qf.binding.QfLora
    def lora(b=0x5000, a=0x6000, rank=16, scale=1.0):
        arr = (L * 1)()
        arr[0].b, arr[0].a, arr[0].rank, arr[0].scale = b, a, rank, scale
        return arr
    t = _tensor(qf, cols=64)
    assert lib.qf_fakequant_lora(2, t, lora(), 1, None, 0, None, None) == UNSUP     # Q4_K not fused
    assert lib.qf_fakequant_lora(1, t, lora(rank=0), 1, None, 0, None, None) == INV
    assert lib.qf_fakequant_lora(1, t, lora(rank=33), 1, None, 0, None, None) == INV
    assert lib.qf_fakequant_lora(1, t, lora(a=0), 1, None, 0, None, None) == INV
    assert lib.qf_fakequant_lora(1, t, lora(a=0x6008), 1, None, 0, None, None) == ALIGN
    assert lib.qf_fakequant_lora(1, t, lora(b=0x5001), 1, None, 0, None, None) == ALIGN
    assert lib.qf_fakequant_lora(1, _tensor(qf, cols=48), lora(), 1, None, 0, None, None) == SHAPE
    assert lib.qf_fakequant_lora(1, _tensor(qf, x_type=1), lora(), 1, None, 0, None, None) == UNSUP
    assert lib.qf_fakequant_lora(0, t, lora(), 1, None, 1, None, None) == INV           # no amax
    assert lib.qf_fakequant_lora(1, t, None, 1, None, 0, None, None) == INV
    assert lib.qf_lora_merge(_tensor(qf, y=0), lora(), 1, None) == INV                   # no output
    assert lib.qf_amax_tied_lora(t, lora(), 1, None, 1, None) == INV
    assert lib.qf_amax_tied_lora(_tensor(qf, group=3), lora(), 1, 0x7000, 2, None) == INV
    assert lib.qf_lora_merge(_tensor(qf, rows=0), lora(), 1, None) == 0                 # empty
    one = lib.qf_amax_fakequant_lora
    assert one(t, lora(), 1, None, 1, None, None) == INV                                  # no amax
    assert one(t, lora(), 1, 0x7000, 0, None, None) == INV
    assert one(_tensor(qf, cols=24), lora(), 1, 0x7000, 1, None, None) == SHAPE          # NVFP4: 16 | cols
    assert one(_tensor(qf, group=1), lora(), 1, 0x7000, 1, None, None) == INV
    assert one(_tensor(qf, y=0, codes=0, scales=0), lora(), 1, 0x7000, 1, None, None) == INV
    assert one(t, lora(rank=40), 1, 0x7000, 1, None, None) == INV
