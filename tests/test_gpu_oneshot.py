"""GPU parity of qf_amax_fakequant: NVFP4 tie-group amax and fused fake-quant + pack in
one call, bit for bit against the oracle.

The single-launch path runs the amax pass, a grid-wide barrier and the encode pass
in one cooperative launch when the inputs fit in L2.  Its results must equal the
oracle's tie-group amax and NVFP4 quantizer (QATFactory project page, Method,
"Numerics": one FP32 tensor scale per fused projection group).  They must also equal
the library's two-call sequence.  Each call must leave its workspace zeroed."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import DEV, assert_same, bits, outputs, u8

pytestmark = pytest.mark.gpu


def _run(xs_cpu, groups, n_groups, tracked=None, workspace="auto", want_y=True):
    xs = [x.to(DEV) for x in xs_cpu]
    outs = [outputs("nvfp4", x, want_y=want_y) for x in xs]
    ys = [o[0].view(x.shape) if o[0] else None for o, x in zip(outs, xs)]
    cs = [o[1].view() for o in outs]
    ss = [o[2].view() if o[2] else None for o in outs]
    amax = torch.full((n_groups,), float("nan"), device=DEV)
    so = torch.full((n_groups,), float("nan"), device=DEV)
    tr = None if tracked is None else torch.tensor(tracked, dtype=torch.float32, device=DEV)
    ws = qf.alloc_workspace(n_groups, DEV) if workspace == "auto" else workspace
    qf.qf_amax_fakequant(xs, ys, cs, ss, groups, amax, tracked=tr, group_scale_out=so,
                         workspace=ws)
    torch.cuda.synchronize()
    if ws is not None:
        qf.qf_workspace_check(ws)
        assert int(ws.count_nonzero()) == 0, "workspace not left zeroed"
    for i, o in enumerate(outs):
        for nm, g in zip(("y", "codes", "scales"), o):
            if g is not None:
                g.check(f"tensor {i} {nm}")
    return {"y": [bits(y) if y is not None else None for y in ys], "codes": [u8(c) for c in cs],
            "scales": [u8(s) if s is not None else None for s in ss], "amax": amax.cpu().numpy(), "s_t": so.cpu().numpy(),
            "tracked": None if tr is None else tr.cpu().numpy()}


def _check_oracle(xs_cpu, groups, n_groups, res, tracked=None, label=""):
    cur = oracle.tied_amax(xs_cpu, groups, n_groups)
    assert_same(f"{label} amax", res["amax"].view(np.uint32), cur.view(np.uint32))
    eff = cur if tracked is None else np.maximum(cur, np.asarray(tracked, np.float32))
    if tracked is not None:
        assert_same(f"{label} tracked", res["tracked"].view(np.uint32), eff.view(np.uint32))
    st = np.float32([oracle.nvfp4_tensor_scale(a) for a in eff])
    assert_same(f"{label} s_t", res["s_t"].view(np.uint32), st.view(np.uint32))
    for i, x in enumerate(xs_cpu):
        y, c, s, _ = oracle.nvfp4(x, float(eff[groups[i]]))
        if res["y"][i] is not None:
            assert_same(f"{label}[{i}] y", res["y"][i], y)
        assert_same(f"{label}[{i}] codes", res["codes"][i], c)
        if res["scales"][i] is not None:
            assert_same(f"{label}[{i}] scales", res["scales"][i], s)


def test_weight_4096_single_launch():
    """The 4096 x 4096 NVFP4 weight (33.5 MB of BF16: the single-launch path), whole."""
    wl = workloads.nvfp4_weight()
    res = _run(wl["tensors"], wl["groups"], wl["n_groups"])
    _check_oracle(wl["tensors"], wl["groups"], wl["n_groups"], res, label="w4096")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tied_groups_small(dtype):
    """Q/K/V and gate/up tie groups (rows scaled down, ragged row counts)."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False, dtype=dtype)
    res = _run(wl["tensors"], wl["groups"], wl["n_groups"])
    _check_oracle(wl["tensors"], wl["groups"], wl["n_groups"], res, label=f"tied {dtype}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_near_the_l2_limit(dtype):
    """Inputs close to the single-launch limit of L2 / 3 (BF16: 1/7 of the tied
    projections, 40.7 MB; FP32: 1/14, also 40.7 MB)."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 7 if dtype == "bf16" else 1 / 14, with_grads=False,
                              dtype=dtype)
    res = _run(wl["tensors"], wl["groups"], wl["n_groups"])
    _check_oracle(wl["tensors"], wl["groups"], wl["n_groups"], res, label=f"tied {dtype}")


@pytest.mark.parametrize("scale", [0.5, 4.0])
def test_tracked_amax(scale):
    """Activations: s_t comes from max(tracked, amax), and tracked is updated in place."""
    wl = workloads.nvfp4_activation(rows_scale=1 / 256)
    a = oracle.amax(wl["tensors"][0])
    tracked = [np.float32(a * scale)]
    res = _run(wl["tensors"], wl["groups"], wl["n_groups"], tracked=tracked)
    _check_oracle(wl["tensors"], wl["groups"], wl["n_groups"], res, tracked=tracked,
                  label=f"tracked x{scale}")


def test_moe_experts_one_call():
    """Many tensors (a 384-entry descriptor table) and 256 tie groups in one launch."""
    wl = workloads.moe_experts(n_experts=128, rows_scale=1 / 64)
    res = _run(wl["tensors"], wl["groups"], wl["n_groups"], want_y=False)
    cur = oracle.tied_amax(wl["tensors"], wl["groups"], wl["n_groups"])
    assert_same("moe amax", res["amax"].view(np.uint32), cur.view(np.uint32))
    for i in range(0, len(wl["tensors"]), 37):
        x = wl["tensors"][i]
        _, c, s, _ = oracle.nvfp4(x, float(cur[wl["groups"][i]]))
        assert_same(f"moe[{i}] codes", res["codes"][i], c)
        assert_same(f"moe[{i}] scales", res["scales"][i], s)


def test_edge_cases():
    """An empty tensor, one row of 16, all-zero and subnormal inputs, a group with no tensor."""
    g = torch.Generator().manual_seed(7)
    xs = [torch.zeros(0, 64, dtype=torch.bfloat16),
          (torch.randn(1, 16, generator=g) * 0.1).to(torch.bfloat16),
          torch.zeros(3, 48, dtype=torch.bfloat16),
          (torch.randn(5, 32, generator=g) * 1e-39).to(torch.bfloat16)]
    groups = [0, 1, 2, 3]
    res = _run(xs, groups, 5)
    _check_oracle(xs, groups, 5, res, label="edge")


def test_reuse_and_two_launch_paths_agree():
    """The same workspace serves consecutive calls.  Without a workspace, and for
    inputs beyond the L2 limit, the call makes two launches with the same bytes."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 16, with_grads=False)
    xs, groups, ng = wl["tensors"], wl["groups"], wl["n_groups"]
    ws = qf.alloc_workspace(ng, DEV)
    first = _run(xs, groups, ng, workspace=ws)
    second = _run(xs, groups, ng, workspace=ws)
    plain = _run(xs, groups, ng, workspace=None)
    for other, nm in ((second, "second call"), (plain, "no workspace")):
        for k in ("y", "codes", "scales"):
            for i in range(len(xs)):
                assert_same(f"{nm} {k}[{i}]", other[k][i], first[k][i])
        assert_same(f"{nm} amax", other["amax"].view(np.uint32), first["amax"].view(np.uint32))
    _check_oracle(xs, groups, ng, first, label="tied 1/16")


def test_large_call_matches_two_calls():
    """Inputs above the L2 limit (the full tied projections, 285 MB): the two-launch
    path, compared with qf_amax_tied + qf_fakequant on the device."""
    wl = workloads.nvfp4_tied(with_grads=False)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]

    def outs():
        o = [qf.alloc_outputs("nvfp4", x) for x in xs]
        return [a[0] for a in o], [a[1] for a in o], [a[2] for a in o]

    y1, c1, s1 = outs()
    a1 = torch.empty(ng, device=DEV)
    qf.qf_amax_fakequant(xs, y1, c1, s1, groups, a1, workspace=qf.alloc_workspace(ng, DEV))
    y2, c2, s2 = outs()
    a2 = torch.empty(ng, device=DEV)
    qf.qf_amax_tied(xs, groups, a2)
    qf.qf_fakequant("nvfp4", xs, y2, c2, s2, groups=groups, group_amax=a2)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2)
    for i in range(len(xs)):
        assert torch.equal(y1[i].view(torch.int16), y2[i].view(torch.int16)), i
        assert torch.equal(c1[i], c2[i]) and torch.equal(s1[i], s2[i]), i


def _guarded_call(xs, groups, ng, ws, tracked=None):
    """One qf_amax_fakequant call into fresh guarded outputs (every byte 0xA5 beforehand,
    the FP32 outputs NaN); returns the buffers."""
    outs = [outputs("nvfp4", x) for x in xs]
    amax = torch.full((ng,), float("nan"), device=DEV)
    so = torch.full((ng,), float("nan"), device=DEV)
    qf.qf_amax_fakequant(xs, [o[0].view(x.shape) for o, x in zip(outs, xs)],
                         [o[1].view() for o in outs], [o[2].view() for o in outs], groups, amax,
                         tracked=tracked, group_scale_out=so, workspace=ws)
    return outs, amax, so


def _untouched(outs, amax, so, label):
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        for nm, g in zip(("y", "codes", "scales"), o):
            assert bool((g.raw == 0xA5).all()), f"{label}: tensor {i} {nm} was written"
    assert bool(torch.isnan(amax).all()) and bool(torch.isnan(so).all()), f"{label}: amax / s_t written"


@pytest.mark.parametrize("rows_scale", [1 / 16, 1 / 7])
def test_barrier_timeout_is_reported_and_recovers(rows_scale):
    """The bounded grid barrier runs out with every CTA present (the testing aid makes
    it wait for one CTA more than the grid holds, at most 1000 polls).  Expected: no
    output is written, the error flag is sticky (a second call on the workspace does
    nothing), qf_workspace_check reports QF_ERR_TIMEOUT and clears it, the workspace
    is all zero again, and the next call is bit-exact to the oracle."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 16, with_grads=False)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    ws = qf.alloc_workspace(ng, DEV)
    try:
        qf.qf_test_barrier_timeout(1000)
        outs, amax, so = _guarded_call(xs, groups, ng, ws)
        _untouched(outs, amax, so, "timed-out call")
    finally:
        qf.qf_test_barrier_timeout(0)
    # sticky: this call finds the flag at entry and does no work
    outs2, amax2, so2 = _guarded_call(xs, groups, ng, ws)
    _untouched(outs2, amax2, so2, "call after the timeout")
    assert int(ws[4:].count_nonzero()) == 0, "counters / slots not reset by the timed-out calls"
    with pytest.raises(qf.QfError) as e:
        qf.qf_workspace_check(ws)
    assert e.value.status == 6                           # QF_ERR_TIMEOUT
    assert int(ws.count_nonzero()) == 0, "workspace not zero after the check"
    qf.qf_workspace_check(ws)                            # cleared: QF_OK now
    res = _run(wl["tensors"], groups, ng, workspace=ws)
    _check_oracle(wl["tensors"], groups, ng, res, label="after timeout")


def _nan_case(where):
    wl = workloads.nvfp4_activation(rows_scale=1 / 256)
    x = wl["tensors"][0].clone()
    tracked = [np.float32(1.5)]
    if where == "x":
        x.view(-1)[12345] = float("nan")
    else:
        tracked = [np.float32("nan")]
    return [x], wl["groups"], wl["n_groups"], tracked


@pytest.mark.parametrize("where", ["x", "tracked"])
def test_nan_folds_alike_on_both_paths(where):
    """A NaN in x or in the running amax is outside the formats, but the call gives the
    same bytes whether it takes the single launch or the two launches: both fold the
    running amax as the max of FP32 bit patterns (a NaN running value stays NaN), and
    both take the block maxima of x alike."""
    xs, groups, ng, tracked = _nan_case(where)
    one = _run(xs, groups, ng, tracked=tracked)
    two = _run(xs, groups, ng, tracked=tracked, workspace=None)
    for k in ("y", "codes", "scales"):
        assert_same(f"{where}: {k}", one[k][0], two[k][0])
    for k in ("amax", "s_t", "tracked"):
        assert_same(f"{where}: {k}", one[k].view(np.uint32), two[k].view(np.uint32))
    if where == "tracked":
        assert np.isnan(one["tracked"][0]) and np.isnan(one["s_t"][0])
