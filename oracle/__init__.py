"""The oracle: a plain CPU statement of deployment-aligned simulated quantization.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` import this package.  The product library
(``fp4_fake_quant_b200``) never imports it, and the two share no code.

The arithmetic lives in ``qf_oracle.c`` (scalar C, IEEE binary32, no FMA); this
module compiles it with gcc and exposes it on numpy arrays.  BF16 tensors are
numpy ``uint16`` arrays of bit patterns.

Method source: "QATFactory: A Versatile, Deployment-Aligned Framework for
Quantization-aware Training and Distillation of LLMs", project page, Method
("Framework overview", "Numerics", "QAD", "QARL", "Export") and the
"Supported formats" table.

Parity status of each function is listed in ``PARITY`` below: every function
is pinned by a CPU test against something other than itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qf_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# function -> the CPU pin(s) in tests/ that check it against something other than itself
PARITY = {
    "f32_to_bf16": "ml_dtypes.bfloat16 conversion (boundary patterns of every BF16 value)",
    "f32_to_f16": "numpy float16 conversion (boundary patterns of every FP16 value)",
    "e2m1_from_f32": "ml_dtypes float4_e2m1fn + brute-force nearest grid; exhaustive change points",
    "e4m3_from_f32": "ml_dtypes float8_e4m3fn + brute-force nearest grid; exhaustive change points",
    "mx_exponent": "math.frexp on every BF16 value",
    "amax": "numpy max(abs) over concatenated tensors",
    "nvfp4_quant": "on-grid round trip, symmetry, block locality, brute-force nearest code, decoder",
    "mxfp4_quant": "on-grid round trip, idempotence, symmetry, brute-force nearest code, decoder",
    "q4k_quant": "on-grid round trip, brute-force nearest q, decoder, error bound",
    "q4k_quant (mse fit)": "grid membership + float64 least error over the grid, never worse than "
                           "min/max, on-grid equal to min/max, decoder, lower total error",
    "ste_backward": "identity copy; clipped mask vs brute-force saturation",
    "lora_merge": "exact integer-grid merges vs numpy; zero adapter / zero scale give W; "
                  "float64 reference within one BF16 step; row/column locality",
}


def build(force: bool = False) -> str:
    """Compile qf_oracle.c into liboracle.so (gcc, -O2, no FMA contraction)."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        sig = {
            "qfo_bf16_to_f32": (F, [ctypes.c_uint16]),
            "qfo_f32_to_bf16": (ctypes.c_uint16, [F]),
            "qfo_f16_to_f32": (F, [ctypes.c_uint16]),
            "qfo_f32_to_f16": (ctypes.c_uint16, [F]),
            "qfo_e2m1_to_f32": (F, [ctypes.c_uint8]),
            "qfo_e2m1_from_f32": (ctypes.c_uint8, [F]),
            "qfo_e4m3_to_f32": (F, [ctypes.c_uint8]),
            "qfo_e4m3_from_f32": (ctypes.c_uint8, [F]),
            "qfo_mx_exponent": (ctypes.c_int, [F]),
            "qfo_amax_bf16": (F, [P, I64]),
            "qfo_amax_x": (F, [P, ctypes.c_int, I64]),
            "qfo_nvfp4_quant_x": (None, [P, ctypes.c_int, I64, I64, F, P, P, P, P]),
            "qfo_mxfp4_quant_x": (None, [P, ctypes.c_int, I64, I64, P, P, P]),
            "qfo_q4k_quant_x": (None, [P, ctypes.c_int, I64, I64, P, P]),
            "qfo_q4k_fit_one_x": (None, [P, ctypes.c_int, P, P, P, P, P]),
            "qfo_q4k_quant_fit": (None, [P, ctypes.c_int, ctypes.c_int, I64, I64, P, P]),
            "qfo_q4k_fit_one_fit": (None, [P, ctypes.c_int, ctypes.c_int, P, P, P, P, P]),
            "qfo_q4k_search_scale_one": (F, [P, F, F]),
            "qfo_ste_backward_x": (None, [P, P, I64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int,
                                          I64, F]),
            "qfo_nvfp4_tensor_scale": (F, [F]),
            "qfo_lora_merge": (None, [P, P, P, I64, I64, ctypes.c_int, F, P]),
            "qfo_nvfp4_quant": (None, [P, I64, I64, F, P, P, P, P]),
            "qfo_mxfp4_quant": (None, [P, I64, I64, P, P, P]),
            "qfo_q4k_quant": (None, [P, I64, I64, P, P]),
            "qfo_q4k_fit_one": (None, [P, P, P, P, P, P]),
            "qfo_nvfp4_decode": (None, [P, P, F, I64, P]),
            "qfo_mxfp4_decode": (None, [P, P, I64, P]),
            "qfo_q4k_decode": (None, [P, I64, P]),
            "qfo_ste_backward": (None, [P, P, I64, ctypes.c_int, ctypes.c_int, P, I64, F]),
            "qfo_e2m1_from_f32_array": (None, [P, I64, P]),
            "qfo_e4m3_from_f32_array": (None, [P, I64, P]),
            "qfo_f32_to_bf16_array": (None, [P, I64, P]),
            "qfo_f32_to_f16_array": (None, [P, I64, P]),
            "qfo_change_points": (I64, [ctypes.c_int, ctypes.c_uint32, ctypes.c_uint32,
                                        P, P, I64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """Accept a numpy uint16 array of BF16 bits or a CPU torch bfloat16 tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # the input generators hand out torch bf16 tensors
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def _xin(x):
    """An input tensor and its element type: BF16 (numpy uint16 bits or torch bf16) -> 0,
    FP32 (numpy float32 or torch float32) -> 1."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.float32:
            return np.ascontiguousarray(x), 1
        return _bits(x), 0
    import torch
    if x.dtype == torch.float32:
        assert x.device.type == "cpu"
        return x.contiguous().numpy(), 1
    return _bits(x), 0


# ---------------------------------------------------------------- conversions
def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def f32_to_bf16(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint16)
    _load().qfo_f32_to_bf16_array(_ptr(f), f.size, _ptr(out))
    return out


def f32_to_f16(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint16)
    _load().qfo_f32_to_f16_array(_ptr(f), f.size, _ptr(out))
    return out


def f16_to_f32(h: int) -> float:
    return _load().qfo_f16_to_f32(int(h))


def e2m1_from_f32(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint8)
    _load().qfo_e2m1_from_f32_array(_ptr(f), f.size, _ptr(out))
    return out


def e2m1_to_f32(c: int) -> float:
    return _load().qfo_e2m1_to_f32(int(c))


def e4m3_from_f32(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint8)
    _load().qfo_e4m3_from_f32_array(_ptr(f), f.size, _ptr(out))
    return out


def e4m3_to_f32(c: int) -> float:
    return _load().qfo_e4m3_to_f32(int(c))


def mx_exponent(amax: float) -> int:
    return _load().qfo_mx_exponent(float(amax))


def change_points(which: str, lo: int, hi: int, cap: int = 1 << 18):
    """Exhaustive scan of bit patterns [lo, hi] (one sign) through a conversion.

    Returns (positions, values, total_count) of the patterns where the result
    changes.  ``which`` is one of 'e2m1', 'e4m3', 'bf16', 'f16'."""
    code = {"e2m1": 0, "e4m3": 1, "bf16": 2, "f16": 3}[which]
    pos = np.zeros(cap, np.uint32)
    val = np.zeros(cap, np.uint32)
    n = _load().qfo_change_points(code, lo, hi, _ptr(pos), _ptr(val), cap)
    k = min(n, cap)
    return pos[:k].copy(), val[:k].copy(), n


# ---------------------------------------------------------------- the method
def amax(x) -> float:
    """max |x| of one BF16 or FP32 tensor (FP32)."""
    xb, xt = _xin(x)
    return float(_load().qfo_amax_x(_ptr(xb), xt, xb.size))


def tied_amax(tensors, groups, n_groups: int, tracked=None) -> np.ndarray:
    """Per tie group: the max over its tensors of max|x|; groups without tensors
    give 0.  With ``tracked`` (FP32 per group), returns max(tracked, amax)."""
    out = np.zeros(n_groups, np.float32)
    for t, g in zip(tensors, groups):
        out[g] = max(out[g], np.float32(amax(t)))
    if tracked is not None:
        out = np.maximum(out, np.asarray(tracked, np.float32))
    return out


def nvfp4_tensor_scale(amax_g: float) -> float:
    return float(_load().qfo_nvfp4_tensor_scale(float(amax_g)))


def nvfp4(x, amax_g: float, rows: int | None = None, cols: int | None = None):
    """NVFP4 quantize-dequantize + pack.  Returns (y_bits, codes, scales, s_t)."""
    xb, xt = _xin(x)
    if rows is None:
        rows, cols = xb.shape
    n = rows * cols
    y = np.empty(n, np.uint16)
    codes = np.empty(n // 2, np.uint8)
    scales = np.empty(n // 16, np.uint8)
    st = ctypes.c_float()
    _load().qfo_nvfp4_quant_x(_ptr(xb), xt, rows, cols, float(amax_g), _ptr(y), _ptr(codes),
                              _ptr(scales), ctypes.byref(st))
    return y, codes, scales, float(st.value)


def mxfp4(x, rows: int | None = None, cols: int | None = None):
    """MXFP4 quantize-dequantize + pack.  Returns (y_bits, codes, scales)."""
    xb, xt = _xin(x)
    if rows is None:
        rows, cols = xb.shape
    n = rows * cols
    y = np.empty(n, np.uint16)
    codes = np.empty(n // 2, np.uint8)
    scales = np.empty(n // 32, np.uint8)
    _load().qfo_mxfp4_quant_x(_ptr(xb), xt, rows, cols, _ptr(y), _ptr(codes), _ptr(scales))
    return y, codes, scales


def q4k(x, rows: int | None = None, cols: int | None = None, mse: bool = False):
    """Q4_K quantize-dequantize + pack (min/max fit, or the MSE-searched fit).
    Returns (y_bits, blocks[n/256, 144])."""
    xb, xt = _xin(x)
    if rows is None:
        rows, cols = xb.shape
    n = rows * cols
    y = np.empty(n, np.uint16)
    blocks = np.empty((n // 256) * 144, np.uint8)
    _load().qfo_q4k_quant_fit(_ptr(xb), xt, int(mse), rows, cols, _ptr(y), _ptr(blocks))
    return y, blocks


def q4k_fit_one(x256: np.ndarray, mse: bool = False):
    """Unpacked fit of one super-block: (d_bits, dmin_bits, sc[8], m[8], q[256])."""
    xb, xt = _xin(x256)
    xb = xb.reshape(-1)
    assert xb.size == 256
    d = ctypes.c_uint16()
    dm = ctypes.c_uint16()
    sc = np.empty(8, np.uint8)
    m = np.empty(8, np.uint8)
    q = np.empty(256, np.uint8)
    _load().qfo_q4k_fit_one_fit(_ptr(xb), xt, int(mse), ctypes.byref(d), ctypes.byref(dm),
                                _ptr(sc), _ptr(m), _ptr(q))
    return int(d.value), int(dm.value), sc, m, q


def q4k_search_scale(v32: np.ndarray, hi: float, min_j: float) -> float:
    """The MSE-searched scale of one 32-element sub-block (values as FP32)."""
    v = np.ascontiguousarray(v32, dtype=np.float32)
    assert v.size == 32
    return float(_load().qfo_q4k_search_scale_one(_ptr(v), float(hi), float(min_j)))


def nvfp4_decode(codes, scales, s_t: float, numel: int) -> np.ndarray:
    y = np.empty(numel, np.uint16)
    _load().qfo_nvfp4_decode(_ptr(np.ascontiguousarray(codes)),
                             _ptr(np.ascontiguousarray(scales)), float(s_t), numel, _ptr(y))
    return y


def mxfp4_decode(codes, scales, numel: int) -> np.ndarray:
    y = np.empty(numel, np.uint16)
    _load().qfo_mxfp4_decode(_ptr(np.ascontiguousarray(codes)),
                             _ptr(np.ascontiguousarray(scales)), numel, _ptr(y))
    return y


def q4k_decode(blocks, numel: int) -> np.ndarray:
    y = np.empty(numel, np.uint16)
    _load().qfo_q4k_decode(_ptr(np.ascontiguousarray(blocks)), numel, _ptr(y))
    return y


def lora_merge(w, b, a, scale: float) -> np.ndarray:
    """The BF16 merged weight M = BF16(W + scale * (B @ A)), B @ A accumulated in FP32
    in increasing k.  w: [rows, cols], b: [rows, r], a: [r, cols], all BF16."""
    wb, bb, ab = _bits(w), _bits(b), _bits(a)
    rows, cols = wb.shape
    r = bb.shape[1]
    assert bb.shape[0] == rows and ab.shape == (r, cols)
    m = np.empty((rows, cols), np.uint16)
    _load().qfo_lora_merge(_ptr(wb), _ptr(np.ascontiguousarray(bb)), _ptr(np.ascontiguousarray(ab)),
                           rows, cols, r, float(scale), _ptr(m))
    return m


FORMATS = {"nvfp4": 0, "mxfp4": 1, "q4k": 2, "q4k_mse": 3}


def ste_backward(grad_y, mode: int = 0, fmt: str = "nvfp4", x=None, amax_g: float = 0.0):
    """STE backward: identity (mode 0) or the clipped reading (mode 1)."""
    gy = _bits(grad_y)
    gx = np.empty(gy.size, np.uint16)
    if mode == 0:
        _load().qfo_ste_backward(_ptr(gy), _ptr(gx), gy.size, 0, 0, None, 0, 0.0)
        return gx
    xb, xt = _xin(x)
    cols = xb.shape[-1]
    _load().qfo_ste_backward_x(_ptr(gy), _ptr(gx), gy.size, 1, FORMATS[fmt], _ptr(xb), xt, cols,
                               float(amax_g))
    return gx
