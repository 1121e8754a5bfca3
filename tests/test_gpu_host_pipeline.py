"""The host pipeline (PCIe copies overlapped with the kernels over several streams)
returns exactly what the device path returns, for every format, with many chunks."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
from fp4_fake_quant_b200.host import HostPipeline
import oracle
import workloads
from gpu_helpers import assert_same, bits, compare_full, u8

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k", "q4k_mse"])
def test_host_pipeline_equals_oracle(fmt):
    wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False)
    xs = [t.pin_memory() for t in wl["tensors"]]
    pipe = HostPipeline(fmt, xs, wl["groups"], wl["n_groups"], chunk_bytes=48 << 10,
                        n_streams=3)
    assert len(pipe.work) > 20                                  # really chunked
    for rep in range(2):                                         # repeated runs reuse buffers
        ys, cs, ss = pipe.run()
        torch.cuda.synchronize()
        res = {"y": [bits(y) for y in ys], "codes": [u8(c) for c in cs],
               "scales": [u8(s) if s is not None else None for s in ss]}
        am = oracle.tied_amax(wl["tensors"], wl["groups"], 2) if fmt == "nvfp4" else None
        if fmt == "nvfp4":
            assert_same("pipeline amax", pipe.amax.cpu().numpy().view(np.uint32), am.view(np.uint32))
        compare_full(fmt, wl["tensors"], res, am, wl["groups"], label=f"pipeline {fmt} {rep}")
