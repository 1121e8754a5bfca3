"""The hot-path calls can be captured in a CUDA graph and replayed.

A training step re-quantizes the same weight buffers every iteration.  Captured
once, the amax pass and the fused pass (and a grouped MoE launch) replay with no
host work.  The calls make no host synchronization and no allocation, and take no
decision from device data, so a replay after the inputs change in place gives the
bytes of a direct call on the new inputs."""
import pytest
import torch

import fp4_fake_quant_b200 as qf
import workloads
from gpu_helpers import DEV

pytestmark = pytest.mark.gpu


def _nvfp4_step(xs, groups, amax, outs):
    qf.qf_amax_tied(xs, groups, amax)
    qf.qf_fakequant("nvfp4", xs, [o[0] for o in outs], [o[1] for o in outs],
                    [o[2] for o in outs], groups, amax)


def test_nvfp4_step_replays_from_a_graph():
    wl = workloads.nvfp4_tied(rows_scale=1 / 32, with_grads=False)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    amax = torch.empty(ng, device=DEV)
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                       # warm-up: fills the host-side caches
        _nvfp4_step(xs, groups, amax, outs)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _nvfp4_step(xs, groups, amax, outs)
    for it in range(2):
        # new weights in place, as an optimizer step would write them
        new = workloads.nvfp4_tied(rows_scale=1 / 32, with_grads=False, seed=40 + it)["tensors"]
        for x, n in zip(xs, new):
            x.copy_(n.to(DEV))
        g.replay()
        ref_amax = torch.empty(ng, device=DEV)
        ref = [qf.alloc_outputs("nvfp4", x) for x in xs]
        _nvfp4_step(xs, groups, ref_amax, ref)
        torch.cuda.synchronize()
        assert torch.equal(amax, ref_amax)
        for (y, c, sc), (y2, c2, sc2) in zip(outs, ref):
            assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
            assert torch.equal(c, c2) and torch.equal(sc, sc2)
    del g


def test_grouped_moe_launch_replays_from_a_graph():
    wl = workloads.moe_experts(n_experts=16, rows_scale=1 / 8)
    xs = [x.to(DEV) for x in wl["tensors"]]
    outs = [qf.alloc_outputs("mxfp4", x) for x in xs]
    call = qf.prepare_fakequant("mxfp4", xs, [o[0] for o in outs], [o[1] for o in outs],
                                [o[2] for o in outs])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for x in xs:
        x.mul_(-0.5)
    g.replay()
    ref = [qf.alloc_outputs("mxfp4", x) for x in xs]
    qf.qf_fakequant("mxfp4", xs, [o[0] for o in ref], [o[1] for o in ref], [o[2] for o in ref])
    torch.cuda.synchronize()
    for (y, c, sc), (y2, c2, sc2) in zip(outs, ref):
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
        assert torch.equal(c, c2) and torch.equal(sc, sc2)
    del g
