"""Python binding of libqf.so: argument marshalling only.

Every function here has the name of the C entry point it calls (include/qf.h)
and does nothing but check tensor dtypes/devices, lay out the ``qf_tensor``
array and pass raw device pointers plus the current CUDA stream.  All
arithmetic runs in the library's sm_100a kernels; there is no fallback: if
libqf.so is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqf.so")

QF_NVFP4, QF_MXFP4, QF_Q4K, QF_Q4K_MSE = 0, 1, 2, 3
QF_X_BF16, QF_X_F32 = 0, 1
FORMATS = {"nvfp4": QF_NVFP4, "mxfp4": QF_MXFP4, "q4k": QF_Q4K, "q4k_mse": QF_Q4K_MSE}
BLOCK = {QF_NVFP4: 16, QF_MXFP4: 32, QF_Q4K: 256, QF_Q4K_MSE: 256}
STATUS = {0: "QF_OK", 1: "QF_ERR_INVALID_ARG", 2: "QF_ERR_SHAPE", 3: "QF_ERR_ALIGN",
          4: "QF_ERR_UNSUPPORTED", 5: "QF_ERR_CUDA", 6: "QF_ERR_TIMEOUT"}


class QfTensor(ctypes.Structure):
    """Mirror of ``qf_tensor`` (include/qf.h)."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("group", ctypes.c_int32), ("x_type", ctypes.c_int32),
                ("y", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class QfLora(ctypes.Structure):
    """Mirror of ``qf_lora`` (include/qf.h)."""
    _fields_ = [("b", ctypes.c_void_p), ("a", ctypes.c_void_p), ("rank", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class QfError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqf.so not built ({LIB_PATH}); run `python -m fp4_fake_quant_b200._build`"
                          " or __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    T = ctypes.POINTER(QfTensor)
    lib.qf_amax_tied.argtypes = [T, I, P, I, P, P]
    lib.qf_fakequant.argtypes = [I, T, I, P, I, P, P]
    lib.qf_pack.argtypes = [I, T, I, P, I, P, P]
    lib.qf_ste_backward.argtypes = [I, P, P, I64, I, T, P, I, P]
    L = ctypes.POINTER(QfLora)
    lib.qf_lora_merge.argtypes = [T, L, I, P]
    lib.qf_amax_tied_lora.argtypes = [T, L, I, P, I, P]
    lib.qf_fakequant_lora.argtypes = [I, T, L, I, P, I, P, P]
    lib.qf_amax_fakequant_lora.argtypes = [T, L, I, P, I, P, P]
    lib.qf_amax_fakequant.argtypes = [T, I, P, I, P, P, P, ctypes.c_size_t, P]
    lib.qf_amax_fakequant_workspace_bytes.argtypes = [I]
    lib.qf_amax_fakequant_workspace_bytes.restype = ctypes.c_size_t
    lib.qf_workspace_check.argtypes = [P, P]
    lib.qf_amax_fakequant_noalloc.argtypes = [T, I, P, I, P, P, P]
    lib.qf_noalloc_check.argtypes = [P]
    lib.qf_test_barrier_timeout.argtypes = [ctypes.c_uint]
    lib.qf_test_barrier_timeout.restype = None
    for f in (lib.qf_amax_tied, lib.qf_fakequant, lib.qf_pack, lib.qf_ste_backward,
              lib.qf_lora_merge, lib.qf_amax_tied_lora, lib.qf_fakequant_lora,
              lib.qf_amax_fakequant, lib.qf_workspace_check, lib.qf_amax_fakequant_noalloc,
              lib.qf_amax_fakequant_lora, lib.qf_noalloc_check):
        f.restype = I
    lib.qf_status_string.argtypes = [I]
    lib.qf_status_string.restype = ctypes.c_char_p
    lib.qf_last_error.argtypes = []
    lib.qf_last_error.restype = ctypes.c_char_p
    lib.qf_version.argtypes = []
    lib.qf_version.restype = I
    return lib


lib = _load()

# the entry points declared in include/qf.h
EXPORTS = ("qf_amax_tied", "qf_fakequant", "qf_pack", "qf_ste_backward", "qf_lora_merge",
           "qf_amax_tied_lora", "qf_fakequant_lora", "qf_amax_fakequant_lora",
           "qf_amax_fakequant", "qf_amax_fakequant_workspace_bytes", "qf_workspace_check",
           "qf_amax_fakequant_noalloc", "qf_noalloc_check", "qf_test_barrier_timeout",
           "qf_status_string", "qf_last_error", "qf_version")


def _check(status: int) -> None:
    if status != 0:
        raise QfError(status, lib.qf_last_error().decode())


def _fmt(f) -> int:
    return FORMATS[f] if isinstance(f, str) else int(f)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libqf must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libqf must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _desc(xs: Sequence[torch.Tensor], ys=None, codes=None, scales=None, groups=None):
    n = len(xs)
    arr = (QfTensor * max(n, 1))()
    for i, x in enumerate(xs):
        if x.dtype == torch.bfloat16:
            xt = QF_X_BF16
        elif x.dtype == torch.float32:
            xt = QF_X_F32
        else:
            raise TypeError("x must be bfloat16 or float32")
        rows, cols = (x.shape[0], x.shape[1]) if x.dim() == 2 else (1, x.numel()) if x.dim() == 1 \
            else (x.numel() // x.shape[-1], x.shape[-1])
        d = arr[i]
        d.x = _ptr(x)
        d.rows, d.cols = rows, cols
        d.group = int(groups[i]) if groups is not None else 0
        d.x_type = xt
        d.y = _ptr(ys[i]) if ys is not None and ys[i] is not None else None
        d.codes = _ptr(codes[i]) if codes is not None and codes[i] is not None else None
        d.scales = _ptr(scales[i]) if scales is not None and scales[i] is not None else None
    return arr, n


def output_sizes(fmt, numel: int):
    """Bytes of (codes, scales) for one tensor of ``numel`` elements."""
    f = _fmt(fmt)
    if f in (QF_Q4K, QF_Q4K_MSE):
        return (numel // 256) * 144, 0
    return numel // 2, numel // BLOCK[f]


def alloc_outputs(fmt, x: torch.Tensor, want_y: bool = True):
    """Allocate (y, codes, scales) for one input tensor (torch allocations; plumbing)."""
    ncodes, nscales = output_sizes(fmt, x.numel())
    y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if want_y else None
    codes = torch.empty(ncodes, dtype=torch.uint8, device=x.device)
    scales = torch.empty(nscales, dtype=torch.uint8, device=x.device) if nscales else None
    return y, codes, scales


def qf_amax_tied(xs: Sequence[torch.Tensor], groups: Sequence[int], group_amax: torch.Tensor,
                 tracked: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    arr, n = _desc(xs, groups=groups)
    _check(lib.qf_amax_tied(arr, n, _ptr(group_amax), group_amax.numel(), _ptr(tracked),
                            _stream(stream)))
    return group_amax


def qf_fakequant(fmt, xs: Sequence[torch.Tensor], ys=None, codes=None, scales=None, groups=None,
                 group_amax: Optional[torch.Tensor] = None,
                 group_scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    arr, n = _desc(xs, ys, codes, scales, groups)
    ng = group_amax.numel() if group_amax is not None else 0
    _check(lib.qf_fakequant(_fmt(fmt), arr, n, _ptr(group_amax), ng, _ptr(group_scale_out),
                            _stream(stream)))


def qf_pack(fmt, xs: Sequence[torch.Tensor], codes, scales=None, groups=None,
            group_amax: Optional[torch.Tensor] = None,
            group_scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    arr, n = _desc(xs, None, codes, scales, groups)
    ng = group_amax.numel() if group_amax is not None else 0
    _check(lib.qf_pack(_fmt(fmt), arr, n, _ptr(group_amax), ng, _ptr(group_scale_out),
                       _stream(stream)))


def qf_ste_backward(grad_y: torch.Tensor, grad_x: torch.Tensor, mode: int = 0, fmt="nvfp4",
                    x: Optional[torch.Tensor] = None, group: int = 0,
                    group_amax: Optional[torch.Tensor] = None, stream=None) -> None:
    fwd = None
    if mode == 1:
        arr, _ = _desc([x], groups=[group])
        fwd = arr
    ng = group_amax.numel() if group_amax is not None else 0
    _check(lib.qf_ste_backward(_fmt(fmt), _ptr(grad_y), _ptr(grad_x), grad_y.numel(), mode, fwd,
                               _ptr(group_amax), ng, _stream(stream)))


class Prepared:
    """A call whose ``qf_tensor`` array and pointers are marshalled once.

    Training loops re-quantize the same weight buffers every step; a prepared call
    skips rebuilding the descriptor array (which for a grouped launch over hundreds
    of MoE expert tensors costs more host time than the kernel takes).  The tensors
    are kept alive by this object; calling it enqueues the same C entry point on
    the current (or given) stream."""

    def __init__(self, fn, args_before_stream, keep):
        self._fn = fn
        self._args = args_before_stream
        self._keep = keep

    def __call__(self, stream=None) -> None:
        _check(self._fn(*self._args, _stream(stream)))


def prepare_fakequant(fmt, xs, ys=None, codes=None, scales=None, groups=None, group_amax=None,
                      group_scale_out=None, pack_only: bool = False) -> Prepared:
    arr, n = _desc(xs, None if pack_only else ys, codes, scales, groups)
    ng = group_amax.numel() if group_amax is not None else 0
    fn = lib.qf_pack if pack_only else lib.qf_fakequant
    keep = (arr, list(xs), ys, codes, scales, group_amax, group_scale_out)
    return Prepared(fn, (_fmt(fmt), arr, n, _ptr(group_amax), ng, _ptr(group_scale_out)), keep)


def prepare_amax_tied(xs, groups, group_amax, tracked=None) -> Prepared:
    arr, n = _desc(xs, groups=groups)
    keep = (arr, list(xs), group_amax, tracked)
    return Prepared(lib.qf_amax_tied, (arr, n, _ptr(group_amax), group_amax.numel(), _ptr(tracked)),
                    keep)


def workspace_bytes(n_groups: int) -> int:
    """Bytes of device workspace qf_amax_fakequant needs for ``n_groups`` tie groups."""
    return int(lib.qf_amax_fakequant_workspace_bytes(int(n_groups)))


def alloc_workspace(n_groups: int, device=None) -> torch.Tensor:
    """A zeroed qf_amax_fakequant workspace (a torch allocation; plumbing)."""
    dev = torch.device(device) if device is not None else torch.device("cuda")
    return torch.zeros(workspace_bytes(n_groups), dtype=torch.uint8, device=dev)


def qf_amax_fakequant(xs, ys=None, codes=None, scales=None, groups=None, group_amax=None,
                      tracked=None, group_scale_out=None, workspace=None, stream=None) -> None:
    """NVFP4 tie-group amax and fused fake-quant + pack in one call (one launch when
    the inputs fit in L2 and a workspace is given)."""
    arr, n = _desc(xs, ys, codes, scales, groups)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.qf_amax_fakequant(arr, n, _ptr(group_amax), group_amax.numel(), _ptr(tracked),
                                 _ptr(group_scale_out), _ptr(workspace), wsb, _stream(stream)))


def prepare_amax_fakequant(xs, ys=None, codes=None, scales=None, groups=None, group_amax=None,
                           tracked=None, group_scale_out=None, workspace=None) -> "Prepared":
    arr, n = _desc(xs, ys, codes, scales, groups)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    keep = (arr, list(xs), ys, codes, scales, group_amax, tracked, group_scale_out, workspace)
    return Prepared(lib.qf_amax_fakequant,
                    (arr, n, _ptr(group_amax), group_amax.numel(), _ptr(tracked),
                     _ptr(group_scale_out), _ptr(workspace), wsb), keep)


def qf_amax_fakequant_noalloc(xs, ys=None, codes=None, scales=None, groups=None,
                              group_amax=None, tracked=None, group_scale_out=None,
                              stream=None) -> None:
    """qf_amax_fakequant on the library's static device workspace (nothing allocated)."""
    arr, n = _desc(xs, ys, codes, scales, groups)
    _check(lib.qf_amax_fakequant_noalloc(arr, n, _ptr(group_amax), group_amax.numel(),
                                         _ptr(tracked), _ptr(group_scale_out), _stream(stream)))


def qf_workspace_check(workspace: torch.Tensor, stream=None) -> None:
    """Synchronize, clear the workspace's error flags, and raise QfError(QF_ERR_TIMEOUT)
    if a grid barrier gave up."""
    _check(lib.qf_workspace_check(_ptr(workspace), _stream(stream)))


def qf_noalloc_check(stream=None) -> None:
    """qf_workspace_check for the static workspace of qf_amax_fakequant_noalloc."""
    _check(lib.qf_noalloc_check(_stream(stream)))


def qf_test_barrier_timeout(polls: int) -> None:
    """Testing aid: with polls > 0 the single-launch grid barrier waits for one CTA
    more than exist and gives up after `polls` polls; 0 restores normal operation."""
    lib.qf_test_barrier_timeout(int(polls))


def _lora(adapters):
    """adapters: sequence of (b [rows, r] BF16, a [r, cols] BF16, scale)."""
    arr = (QfLora * max(len(adapters), 1))()
    for i, (b, a, scale) in enumerate(adapters):
        if b.dtype != torch.bfloat16 or a.dtype != torch.bfloat16:
            raise TypeError("LoRA factors must be bfloat16")
        arr[i].b = _ptr(b)
        arr[i].a = _ptr(a)
        arr[i].rank = int(a.shape[0])
        arr[i].scale = float(scale)
    return arr


def qf_lora_merge(xs, adapters, merged, stream=None) -> None:
    """merged[i] <- BF16(xs[i] + scale * b @ a), b @ a accumulated in FP32 in increasing k."""
    arr, n = _desc(xs, merged)
    _check(lib.qf_lora_merge(arr, _lora(adapters), n, _stream(stream)))


def qf_amax_tied_lora(xs, adapters, groups, group_amax, stream=None):
    arr, n = _desc(xs, groups=groups)
    _check(lib.qf_amax_tied_lora(arr, _lora(adapters), n, _ptr(group_amax), group_amax.numel(),
                                 _stream(stream)))
    return group_amax


def qf_fakequant_lora(fmt, xs, adapters, ys=None, codes=None, scales=None, groups=None,
                      group_amax=None, group_scale_out=None, stream=None) -> None:
    arr, n = _desc(xs, ys, codes, scales, groups)
    ng = group_amax.numel() if group_amax is not None else 0
    _check(lib.qf_fakequant_lora(_fmt(fmt), arr, _lora(adapters), n, _ptr(group_amax), ng,
                                 _ptr(group_scale_out), _stream(stream)))


def qf_amax_fakequant_lora(xs, adapters, ys=None, codes=None, scales=None, groups=None,
                           group_amax=None, group_scale_out=None, stream=None) -> None:
    """LoRA-QAD NVFP4 step: merged-weight group amax, then fake-quant + pack (one call)."""
    arr, n = _desc(xs, ys, codes, scales, groups)
    _check(lib.qf_amax_fakequant_lora(arr, _lora(adapters), n, _ptr(group_amax),
                                      group_amax.numel(), _ptr(group_scale_out), _stream(stream)))


def prepare_amax_fakequant_lora(xs, adapters, ys=None, codes=None, scales=None, groups=None,
                                group_amax=None, group_scale_out=None) -> "Prepared":
    arr, n = _desc(xs, ys, codes, scales, groups)
    la = _lora(adapters)
    keep = (arr, la, list(xs), list(adapters), ys, codes, scales, group_amax, group_scale_out)
    return Prepared(lib.qf_amax_fakequant_lora,
                    (arr, la, n, _ptr(group_amax), group_amax.numel(), _ptr(group_scale_out)), keep)


def prepare_fakequant_lora(fmt, xs, adapters, ys=None, codes=None, scales=None, groups=None,
                           group_amax=None, group_scale_out=None) -> "Prepared":
    arr, n = _desc(xs, ys, codes, scales, groups)
    la = _lora(adapters)
    ng = group_amax.numel() if group_amax is not None else 0
    keep = (arr, la, list(xs), list(adapters), ys, codes, scales, group_amax, group_scale_out)
    return Prepared(lib.qf_fakequant_lora, (_fmt(fmt), arr, la, n, _ptr(group_amax), ng,
                                            _ptr(group_scale_out)), keep)


def prepare_amax_tied_lora(xs, adapters, groups, group_amax) -> "Prepared":
    arr, n = _desc(xs, groups=groups)
    la = _lora(adapters)
    keep = (arr, la, list(xs), list(adapters), group_amax)
    return Prepared(lib.qf_amax_tied_lora, (arr, la, n, _ptr(group_amax), group_amax.numel()), keep)
