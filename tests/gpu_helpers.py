"""Shared helpers for the GPU parity tests: run the CUDA path through the binding
and compare its bytes with the oracle's.  Bit-exact comparisons only."""
from __future__ import annotations

import os

import numpy as np
import torch

import fp4_fake_quant_b200 as qf
import oracle

DEV = "cuda:0"
GUARD = 64          # bytes of guard after every output buffer
PATTERN = 0xA5


def bits(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor (any device) -> numpy uint16 bit patterns, flat."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().reshape(-1)


def assert_same(name: str, got: np.ndarray, want: np.ndarray) -> None:
    got = np.asarray(got).reshape(-1)
    want = np.asarray(want).reshape(-1)
    assert got.shape == want.shape, f"{name}: shape {got.shape} vs {want.shape}"
    if not np.array_equal(got, want):
        bad = np.nonzero(got != want)[0]
        i = int(bad[0])
        raise AssertionError(f"{name}: {bad.size} of {got.size} differ; first at {i}: "
                             f"got {int(got[i]):#x} want {int(want[i]):#x}")


class Guarded:
    """An output buffer with GUARD bytes of a known pattern after it."""

    def __init__(self, nbytes: int, dtype=torch.uint8, device=DEV):
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.dtype = dtype

    def view(self, shape=None) -> torch.Tensor:
        t = self.raw[: self.nbytes].view(self.dtype)
        return t.view(shape) if shape is not None else t

    def check(self, name: str) -> None:
        tail = self.raw[self.nbytes:].cpu().numpy()
        assert np.all(tail == PATTERN), f"{name}: wrote past the end of its buffer"


def outputs(fmt: str, x: torch.Tensor, want_y: bool = True):
    """Guarded (y, codes, scales) for one input."""
    ncodes, nscales = qf.output_sizes(fmt, x.numel())
    y = Guarded(x.numel() * 2, torch.bfloat16) if want_y else None
    c = Guarded(ncodes)
    s = Guarded(nscales) if nscales else None
    return y, c, s


def run_fakequant(fmt: str, xs_cpu, groups=None, n_groups: int = 1, tracked=None,
                  pack_only: bool = False):
    """Run the CUDA path on CPU bf16 tensors.  NVFP4 runs qf_amax_tied first.
    Returns dict with per-tensor numpy outputs and (NVFP4) amax / s_t."""
    xs = [x.to(DEV) for x in xs_cpu]
    groups = list(groups) if groups is not None else [0] * len(xs)
    res = {}
    so = None
    q_amax = None          # the amax the quantization uses: the group amax, or the tracked one
    if fmt == "nvfp4":
        amax = torch.full((n_groups,), float("nan"), dtype=torch.float32, device=DEV)
        tr = None if tracked is None else torch.as_tensor(tracked, dtype=torch.float32).to(DEV)
        qf.qf_amax_tied(xs, groups, amax, tracked=tr)
        so = torch.full((n_groups,), float("nan"), dtype=torch.float32, device=DEV)
        q_amax = tr if tr is not None else amax
        res["amax"] = amax.cpu().numpy()
    outs = [outputs(fmt, x, want_y=not pack_only) for x in xs]
    ys = [o[0].view(x.shape) if o[0] else None for o, x in zip(outs, xs)]
    cs = [o[1].view() for o in outs]
    ss = [o[2].view() if o[2] else None for o in outs]
    if pack_only:
        qf.qf_pack(fmt, xs, cs, ss, groups=groups,
                   group_amax=q_amax, group_scale_out=so)
    else:
        qf.qf_fakequant(fmt, xs, ys, cs, ss, groups=groups, group_amax=q_amax,
                        group_scale_out=so)
    torch.cuda.synchronize()
    if fmt == "nvfp4":
        res["s_t"] = so.cpu().numpy()
        if tracked is not None:
            res["tracked"] = q_amax.cpu().numpy()
    res["y"] = [bits(y) if y is not None else None for y in ys]
    res["codes"] = [u8(c) for c in cs]
    res["scales"] = [u8(s) if s is not None else None for s in ss]
    for i, o in enumerate(outs):
        for nm, g in zip(("y", "codes", "scales"), o):
            if g is not None:
                g.check(f"tensor {i} {nm}")
    return res


def oracle_outputs(fmt: str, x_cpu, amax_g: float = 0.0):
    """Oracle (y, codes, scales) of one whole tensor."""
    if fmt == "nvfp4":
        y, c, s, _ = oracle.nvfp4(x_cpu, amax_g)
        return y, c, s
    if fmt == "mxfp4":
        return oracle.mxfp4(x_cpu)
    y, b = oracle.q4k(x_cpu, mse=fmt == "q4k_mse")
    return y, b, None


def compare_full(fmt: str, xs_cpu, res, amax=None, groups=None, label=""):
    groups = groups or [0] * len(xs_cpu)
    for i, x in enumerate(xs_cpu):
        a = float(amax[groups[i]]) if amax is not None else 0.0
        y, c, s = oracle_outputs(fmt, x, a)
        if res["y"][i] is not None:
            assert_same(f"{label}[{i}] y", res["y"][i], y)
        assert_same(f"{label}[{i}] codes", res["codes"][i], c)
        if s is not None and res["scales"][i] is not None:
            assert_same(f"{label}[{i}] scales", res["scales"][i], s)


def compare_rows(fmt: str, x_cpu, y_bits, codes, scales, rows, amax_g: float = 0.0, label=""):
    """Compare the CUDA outputs of selected rows with the oracle run on those rows alone
    (rows are independent given the tie-group amax)."""
    R, K = x_cpu.shape
    q4 = fmt in ("q4k", "q4k_mse")
    cpr = K // 2 if not q4 else (K // 256) * 144
    spr = K // (16 if fmt == "nvfp4" else 32) if not q4 else 0
    for r in rows:
        xr = x_cpu[r:r + 1]
        y, c, s = oracle_outputs(fmt, xr, amax_g)
        if y_bits is not None:
            assert_same(f"{label} row {r} y", y_bits[r * K:(r + 1) * K], y)
        assert_same(f"{label} row {r} codes", codes[r * cpr:(r + 1) * cpr], c)
        if spr and scales is not None:
            assert_same(f"{label} row {r} scales", scales[r * spr:(r + 1) * spr], s)


def sample_rows(R: int, k: int, seed: int):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(R, size=min(k, R), replace=False).tolist())
    rows |= {0, R - 1}
    return sorted(rows)


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def row_parts(n_rows: int, parts: int):
    cuts = [n_rows * i // parts for i in range(parts + 1)]
    return [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]


def oracle_whole(fmt: str, x_cpu, amax_g: float = 0.0, pool=None):
    """The oracle's (y, codes, scales) of one whole tensor, its rows split into ranges
    that run on host threads (the oracle's C calls release the GIL; rows are
    independent given the tie-group amax, and every output is in flat row order, so
    the concatenation is the one-call result)."""
    if pool is None:
        return oracle_outputs(fmt, x_cpu, amax_g)
    parts = list(pool.map(lambda ab: oracle_outputs(fmt, x_cpu[ab[0]:ab[1]], amax_g),
                          row_parts(x_cpu.shape[0], host_threads())))
    cat = lambda k: None if parts[0][k] is None else np.concatenate([p[k] for p in parts])  # noqa: E731
    return cat(0), cat(1), cat(2)
