"""Fake-quant of host-resident tensors with the PCIe copies overlapped.

Quantizing weights that live in host memory (a checkpoint export, a weight sync
from a CPU copy) is bound by the host<->device link, not by the kernels.  This
helper splits every tensor into row chunks (rows are independent in every format)
and spreads the chunks over several CUDA streams: the host->device copy of one
chunk, the fused kernel of another and the device->host copy of a third run at
the same time, and both copy directions are busy at once.

NVFP4 needs each tie group's amax before any block is encoded, so its inputs are
first streamed in while qf_amax_tied accumulates the running amax per chunk
(its tracked-maximum form), then the encode and the copies out are pipelined.

All kernels are the library's (through the C ABI); this module only orders
copies and launches on streams.  Host tensors must be pinned for the copies to
be asynchronous.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import binding as B


def _chunks(rows: int, cols: int, elem_bytes: int, target_bytes: int):
    per = max(1, target_bytes // max(1, cols * elem_bytes))
    r = 0
    while r < rows:
        yield r, min(rows, r + per)
        r += per


class HostPipeline:
    """Prepared host->device->host fake-quant of a fixed set of tensors.

    xs_host: pinned CPU inputs (BF16 or FP32, 2-D); the device copies, the device
    outputs and the pinned host outputs are allocated once here.  run() performs
    one full pass and returns the host outputs (y, codes, scales per tensor)."""

    def __init__(self, fmt, xs_host: Sequence[torch.Tensor], groups: Optional[Sequence[int]] = None,
                 n_groups: int = 1, device=None, want_y: bool = True, chunk_bytes: int = 24 << 20,
                 n_streams: int = 3):
        self.fmt = B._fmt(fmt)
        self.dev = torch.device(device) if device is not None else torch.device("cuda")
        self.xs_h = list(xs_host)
        self.xs_d = [torch.empty_like(x, device=self.dev) for x in self.xs_h]
        outs = [B.alloc_outputs(fmt, x, want_y) for x in self.xs_d]
        self.ys_d = [o[0] for o in outs]
        self.cs_d = [o[1] for o in outs]
        self.ss_d = [o[2] for o in outs]
        pin = lambda t: None if t is None else torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
        self.ys_h = [pin(t) for t in self.ys_d]
        self.cs_h = [pin(t) for t in self.cs_d]
        self.ss_h = [pin(t) for t in self.ss_d]
        self.groups = list(groups) if groups is not None else [0] * len(self.xs_h)
        self.nv = self.fmt == B.QF_NVFP4
        self.streams = [torch.cuda.Stream(device=self.dev) for _ in range(n_streams)]
        if self.nv:
            # the running (tracked) max is updated with atomics from every stream; each
            # stream has its own per-chunk amax output
            self.amax = torch.zeros(n_groups, dtype=torch.float32, device=self.dev)
            self.chunk_amax = [torch.zeros(n_groups, dtype=torch.float32, device=self.dev)
                               for _ in self.streams]
        # (tensor, row0, row1) chunks and their prepared kernel calls
        self.work = []
        for i, x in enumerate(self.xs_h):
            rows, cols = x.shape
            for r0, r1 in _chunks(rows, cols, x.element_size(), chunk_bytes):
                self.work.append((i, r0, r1))
        self._fq = []
        self._am = []
        for k, (i, r0, r1) in enumerate(self.work):
            cols = self.xs_h[i].shape[1]
            xd = self.xs_d[i][r0:r1]
            y = self.ys_d[i][r0:r1] if self.ys_d[i] is not None else None
            c = self._rows_of(self.cs_d[i], r0, r1, cols, codes=True)
            s = self._rows_of(self.ss_d[i], r0, r1, cols, codes=False)
            kw = {}
            if self.nv:
                kw = {"groups": [self.groups[i]], "group_amax": self.amax}
                self._am.append(B.prepare_amax_tied(
                    [xd], [self.groups[i]], self.chunk_amax[k % len(self.streams)],
                    tracked=self.amax))
            self._fq.append(B.prepare_fakequant(fmt, [xd], [y], [c], [s], **kw))

    def _rows_of(self, t, r0, r1, cols, codes):
        """The slice of a flat codes / scales buffer that holds rows [r0, r1)."""
        if t is None:
            return None
        if codes:
            b = (cols // 256) * 144 if self.fmt in (B.QF_Q4K, B.QF_Q4K_MSE) else cols // 2
        else:
            b = cols // B.BLOCK[self.fmt]
        return t[r0 * b:r1 * b]

    def run(self):
        cur = torch.cuda.current_stream(self.dev)
        if self.nv:
            self.amax.zero_()
        for st in self.streams:
            st.wait_stream(cur)
        if self.nv:
            # pass 1: stream the inputs in; each chunk's amax folds into the running max
            for k, (i, r0, r1) in enumerate(self.work):
                st = self.streams[k % len(self.streams)]
                with torch.cuda.stream(st):
                    self.xs_d[i][r0:r1].copy_(self.xs_h[i][r0:r1], non_blocking=True)
                    self._am[k](st)
            # every encode needs the final amax of its group
            for a in self.streams:
                for b in self.streams:
                    if a is not b:
                        a.wait_stream(b)
        for k, (i, r0, r1) in enumerate(self.work):
            st = self.streams[k % len(self.streams)]
            with torch.cuda.stream(st):
                if not self.nv:
                    self.xs_d[i][r0:r1].copy_(self.xs_h[i][r0:r1], non_blocking=True)
                self._fq[k](st)
                cols = self.xs_h[i].shape[1]
                if self.ys_d[i] is not None:
                    self.ys_h[i][r0:r1].copy_(self.ys_d[i][r0:r1], non_blocking=True)
                c_d = self._rows_of(self.cs_d[i], r0, r1, cols, True)
                c_h = self._rows_of(self.cs_h[i], r0, r1, cols, True)
                c_h.copy_(c_d, non_blocking=True)
                if self.ss_d[i] is not None:
                    self._rows_of(self.ss_h[i], r0, r1, cols, False).copy_(
                        self._rows_of(self.ss_d[i], r0, r1, cols, False), non_blocking=True)
        for st in self.streams:
            cur.wait_stream(st)
        return self.ys_h, self.cs_h, self.ss_h

    @property
    def h2d_bytes(self) -> int:
        return sum(x.numel() * x.element_size() for x in self.xs_h)

    @property
    def d2h_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.ys_h + self.cs_h + self.ss_h
                   if t is not None)
