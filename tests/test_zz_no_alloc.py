"""qf_amax_fakequant_noalloc: the one-shot NVFP4 call on the library's static device
workspace gives, through the C ABI, the same bytes as qf_amax_fakequant with a
caller workspace.  Both are called twice in a row on the same inputs.

The file sorts last so that it also runs after every other GPU test has used the
device; it passes alone as well."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import DEV, assert_same, bits, u8

MAX_GROUPS = 4092


def test_oversize_is_rejected_before_any_launch():
    """Host-side checks only: no device memory is touched."""
    lib = qf.lib
    arr = (qf.binding.QfTensor * 1)()
    assert lib.qf_amax_fakequant_noalloc(arr, 1, 0x5000, MAX_GROUPS + 1, None, None, None) == 1
    assert b"static workspace" in lib.qf_last_error()
    assert lib.qf_amax_fakequant_noalloc(arr, 1, 0x5000, 0, None, None, None) == 1
    assert lib.qf_amax_fakequant_noalloc(None, 1, 0x5000, 1, None, None, None) == 1


def _outs(xs):
    o = [qf.alloc_outputs("nvfp4", x) for x in xs]
    return [a[0] for a in o], [a[1] for a in o], [a[2] for a in o]


def _snapshot(ys, cs, ss, amax, so):
    return ([bits(y) for y in ys], [u8(c) for c in cs], [u8(s) for s in ss],
            amax.cpu().numpy().view(np.uint32).copy(), so.cpu().numpy().view(np.uint32).copy())


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["weight_4096", "tied_small", "moe_small"])
def test_noalloc_matches_workspace_call_twice(case):
    if case == "weight_4096":
        wl = workloads.nvfp4_weight()
    elif case == "tied_small":
        wl = workloads.nvfp4_tied(rows_scale=1 / 32, with_grads=False)
    else:
        wl = workloads.moe_experts(n_experts=32, rows_scale=1 / 16)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    ws = qf.alloc_workspace(ng, DEV)
    ref, got = [], []
    for _ in range(2):
        ys, cs, ss = _outs(xs)
        amax, so = torch.empty(ng, device=DEV), torch.empty(ng, device=DEV)
        qf.qf_amax_fakequant(xs, ys, cs, ss, groups, amax, group_scale_out=so, workspace=ws)
        torch.cuda.synchronize()
        ref.append(_snapshot(ys, cs, ss, amax, so))
        ys, cs, ss = _outs(xs)
        amax, so = torch.empty(ng, device=DEV), torch.empty(ng, device=DEV)
        qf.qf_amax_fakequant_noalloc(xs, ys, cs, ss, groups, amax, group_scale_out=so)
        torch.cuda.synchronize()
        got.append(_snapshot(ys, cs, ss, amax, so))
    for k in range(2):
        for part, nm in zip(range(5), ("y", "codes", "scales", "amax", "s_t")):
            a, b = got[k][part], ref[k][part]
            if isinstance(a, list):
                for i in range(len(a)):
                    assert_same(f"call {k} {nm}[{i}]", a[i], b[i])
            else:
                assert_same(f"call {k} {nm}", a, b)
    # and the group amax is the oracle's
    want = oracle.tied_amax(wl["tensors"], groups, ng)
    assert_same("amax vs oracle", got[1][3], want.view(np.uint32))
