"""Full-size parity, whole: every output byte of every configuration, at the sizes the
benchmark times, against the oracle.

The oracle runs over every row, its rows split into ranges on all host threads
(rows are independent given the tie-group amax, so the bytes are those of one
call).  Configurations: MXFP4 W4A4 (W 12288x4096 + A 32768x4096, one grouped
launch); Q4_K down 4096x14336 + up 14336x4096 (min/max fit, MSE-searched fit, FP32
master weights); NVFP4 tied Q/K/V + gate/up with both STE modes (BF16 and FP32
master weights); MoE 128 experts x (gate, up, down), 384 tensors in one grouped
launch, in all three formats; the NVFP4 activation 32768x4096 with a tracked amax;
and the LoRA-merged NVFP4 step (rank 16) on the tied projections."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import (DEV, assert_same, bits, host_threads, oracle_whole, row_parts,
                         run_fakequant, u8)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def moe():
    return workloads.moe_experts()        # one input set for the three formats


@pytest.fixture(scope="module")
def pool():
    with ThreadPoolExecutor(max_workers=host_threads()) as p:
        yield p


def _check_all(fmt, xs, res, pool, amax=None, groups=None, label=""):
    groups = groups or [0] * len(xs)
    for i, x in enumerate(xs):
        a = float(amax[groups[i]]) if amax is not None else 0.0
        y, c, s = oracle_whole(fmt, x, a, pool)
        assert_same(f"{label}[{i}] y", res["y"][i], y)
        assert_same(f"{label}[{i}] codes", res["codes"][i], c)
        if s is not None:
            assert_same(f"{label}[{i}] scales", res["scales"][i], s)


def test_w4a4_whole(pool):
    wl = workloads.mxfp4_w4a4()
    res = run_fakequant("mxfp4", wl["tensors"])
    _check_all("mxfp4", wl["tensors"], res, pool, label="w4a4")


@pytest.mark.parametrize("fmt,dtype", [("q4k", "bf16"), ("q4k", "f32"), ("q4k_mse", "bf16")])
def test_q4k_whole(pool, fmt, dtype):
    wl = workloads.q4k_weights(dtype=dtype)
    res = run_fakequant(fmt, wl["tensors"])
    _check_all(fmt, wl["tensors"], res, pool, label=f"{fmt} {dtype}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_nvfp4_tied_whole_with_ste(pool, dtype):
    wl = workloads.nvfp4_tied(dtype=dtype, with_grads=dtype == "bf16")
    ts, groups, ng = wl["tensors"], wl["groups"], wl["n_groups"]
    res = run_fakequant("nvfp4", ts, groups, ng)
    am = oracle.tied_amax(ts, groups, ng)
    assert_same("tied amax", res["amax"].view(np.uint32), am.view(np.uint32))
    st = np.float32([oracle.nvfp4_tensor_scale(a) for a in am])
    assert_same("tied s_t", res["s_t"].view(np.uint32), st.view(np.uint32))
    _check_all("nvfp4", ts, res, pool, am, groups, label=f"tied {dtype}")
    if dtype != "bf16":
        return
    # the STE backward of every tensor, identity and clipped, whole
    amax = torch.from_numpy(am).to(DEV)
    for i, (x, gy) in enumerate(zip(ts, wl["grads"])):
        xd, gd = x.to(DEV), gy.to(DEV)
        for mode in (0, 1):
            out = torch.empty_like(gd)
            qf.qf_ste_backward(gd, out, mode, "nvfp4", xd, groups[i], amax)
            torch.cuda.synchronize()
            a = float(am[groups[i]])
            want = np.concatenate(list(pool.map(
                lambda ab: oracle.ste_backward(gy[ab[0]:ab[1]], mode, "nvfp4", x[ab[0]:ab[1]], a),
                row_parts(x.shape[0], host_threads()))))
            assert_same(f"tied STE mode {mode} [{i}]", bits(out), want)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_moe_grouped_whole(pool, moe, fmt):
    """All 384 expert tensors in one grouped launch; every tensor compared whole."""
    wl = moe
    ts, groups, ng = wl["tensors"], wl["groups"], wl["n_groups"]
    res = run_fakequant(fmt, ts, groups, ng)
    am = oracle.tied_amax(ts, groups, ng) if fmt == "nvfp4" else None
    if fmt == "nvfp4":
        assert_same("moe amax", res["amax"].view(np.uint32), am.view(np.uint32))
    want = list(pool.map(lambda i: oracle_whole(fmt, ts[i], float(am[groups[i]]) if am is not None
                                                else 0.0), range(len(ts))))
    for i, (y, c, s) in enumerate(want):
        assert_same(f"moe {fmt} [{i}] y", res["y"][i], y)
        assert_same(f"moe {fmt} [{i}] codes", res["codes"][i], c)
        if s is not None:
            assert_same(f"moe {fmt} [{i}] scales", res["scales"][i], s)


def test_activation_tracked_whole(pool):
    a = workloads.nvfp4_activation()["tensors"][0]
    am = oracle.amax(a)
    res = run_fakequant("nvfp4", [a], tracked=[0.0])
    assert res["tracked"][0] == np.float32(am)
    _check_all("nvfp4", [a], res, pool, np.float32([am]), label="activation")


def test_lora_step_whole(pool):
    """qf_amax_fakequant_lora on the tied projections with rank-16 adapters (scale 2):
    the merged weight of every tensor, its tie-group amax and its NVFP4 outputs."""
    wl = workloads.nvfp4_tied(with_grads=False)
    ts, groups, ng = wl["tensors"], wl["groups"], wl["n_groups"]
    r, scale = 16, 2.0
    ads = [(workloads.normal_with_outliers(x.shape[0], r, 0.01, 0, 1, 9, 2 * i),
            workloads.normal_with_outliers(r, x.shape[1], 0.02, 0, 1, 9, 2 * i + 1))
           for i, x in enumerate(ts)]
    xs = [x.to(DEV) for x in ts]
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    amax = torch.full((ng,), float("nan"), device=DEV)
    so = torch.full((ng,), float("nan"), device=DEV)
    qf.qf_amax_fakequant_lora(xs, [(b.to(DEV), a.to(DEV), scale) for b, a in ads],
                              [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs],
                              groups, amax, so)
    torch.cuda.synchronize()
    merged = []
    for x, (b, a) in zip(ts, ads):
        merged.append(np.concatenate(list(pool.map(
            lambda ab: oracle.lora_merge(x[ab[0]:ab[1]], b[ab[0]:ab[1]], a, scale),
            row_parts(x.shape[0], host_threads())))))
    am = oracle.tied_amax(merged, groups, ng)
    assert_same("lora amax", amax.cpu().numpy().view(np.uint32), am.view(np.uint32))
    st = np.float32([oracle.nvfp4_tensor_scale(v) for v in am])
    assert_same("lora s_t", so.cpu().numpy().view(np.uint32), st.view(np.uint32))
    for i, m in enumerate(merged):
        y, c, s = oracle_whole("nvfp4", m, float(am[groups[i]]), pool)
        assert_same(f"lora [{i}] y", bits(outs[i][0]), y)
        assert_same(f"lora [{i}] codes", u8(outs[i][1]), c)
        assert_same(f"lora [{i}] scales", u8(outs[i][2]), s)
