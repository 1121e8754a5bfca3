"""qf_amax_fakequant_noalloc: the one-shot NVFP4 call on the library's static device
workspace gives, through the C ABI, the same bytes as qf_amax_fakequant with a
caller workspace, and those of the oracle.  Both are called twice in a row on the
same inputs.  A barrier timeout on the static workspace is reported by
qf_noalloc_check.

The file sorts last so that it also runs after every other GPU test has used the
device; it passes alone as well."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import DEV, assert_same, bits, compare_full, u8

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
    qf.qf_noalloc_check()                   # no timeout recorded
    # and every output is the oracle's, byte for byte
    want = oracle.tied_amax(wl["tensors"], groups, ng)
    assert_same("amax vs oracle", got[1][3], want.view(np.uint32))
    st = np.float32([oracle.nvfp4_tensor_scale(a) for a in want])
    assert_same("s_t vs oracle", got[1][4], st.view(np.uint32))
    for k in range(2):
        res = {"y": got[k][0], "codes": got[k][1], "scales": got[k][2]}
        compare_full("nvfp4", wl["tensors"], res, amax=want, groups=groups,
                     label=f"{case} call {k} vs oracle")


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_by_noalloc_check():
    """The barrier of the static-workspace call runs out (testing aid: it waits for one
    CTA more than the grid holds, at most 1000 polls).  No output is written, the
    following call does nothing either, qf_noalloc_check reports QF_ERR_TIMEOUT once,
    and the next call gives the oracle's bytes."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 32, with_grads=False)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    qf.qf_noalloc_check()                   # whatever earlier tests left: start clean

    def call():
        ys, cs, ss = _outs(xs)
        for t in ys + cs + ss:
            t.view(torch.uint8).fill_(0xA5)
        amax = torch.full((ng,), float("nan"), device=DEV)
        qf.qf_amax_fakequant_noalloc(xs, ys, cs, ss, groups, amax)
        torch.cuda.synchronize()
        return ys, cs, ss, amax

    def untouched(r, label):
        ys, cs, ss, amax = r
        for t in ys + cs + ss:
            assert bool((t.view(torch.uint8) == 0xA5).all()), f"{label}: an output was written"
        assert bool(torch.isnan(amax).all()), f"{label}: amax written"

    try:
        qf.qf_test_barrier_timeout(1000)
        untouched(call(), "timed-out call")
    finally:
        qf.qf_test_barrier_timeout(0)
    untouched(call(), "call after the timeout")
    with pytest.raises(qf.QfError) as e:
        qf.qf_noalloc_check()
    assert e.value.status == 6              # QF_ERR_TIMEOUT
    qf.qf_noalloc_check()                   # cleared
    ys, cs, ss, amax = call()
    want = oracle.tied_amax(wl["tensors"], groups, ng)
    assert_same("amax vs oracle", amax.cpu().numpy().view(np.uint32), want.view(np.uint32))
    res = {"y": [bits(y) for y in ys], "codes": [u8(c) for c in cs], "scales": [u8(s) for s in ss]}
    compare_full("nvfp4", wl["tensors"], res, amax=want, groups=groups, label="after timeout")
