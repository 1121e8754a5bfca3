"""GPU parity: the CUDA path (through the C ABI) against the oracle, bit for bit.

Tolerance is 0 ulp for every output: codes, scales, packed bytes, dequantized
BF16, tensor amax / scales and STE gradients.  Small cases (reduced row counts
of the five workloads, ragged and degenerate shapes) are compared whole; the
full-size workloads run in the launch configuration the benchmark times and are
compared on sampled rows, each recomputed by the oracle alone.
"""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import (DEV, Guarded, assert_same, bits, compare_full, compare_rows,
                         run_fakequant, sample_rows, u8)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------- small, whole
@pytest.mark.parametrize("rows_scale", [1 / 64, 1 / 4])
def test_nvfp4_weight(rows_scale):
    wl = workloads.nvfp4_weight(rows_scale=rows_scale)
    res = run_fakequant("nvfp4", wl["tensors"])
    am = oracle.tied_amax(wl["tensors"], [0], 1)
    assert_same("amax", res["amax"].view(np.uint32), am.view(np.uint32))
    st = np.float32(oracle.nvfp4_tensor_scale(am[0]))
    assert_same("s_t", res["s_t"].view(np.uint32), np.array([st]).view(np.uint32))
    compare_full("nvfp4", wl["tensors"], res, am, label="w")


def test_mxfp4_w4a4_small():
    wl = workloads.mxfp4_w4a4(rows_scale=1 / 64)
    res = run_fakequant("mxfp4", wl["tensors"])
    compare_full("mxfp4", wl["tensors"], res, label="w4a4")


def test_q4k_small():
    wl = workloads.q4k_weights(rows_scale=1 / 64)
    res = run_fakequant("q4k", wl["tensors"])
    compare_full("q4k", wl["tensors"], res, label="q4k")


def test_nvfp4_tied_small_with_ste():
    wl = workloads.nvfp4_tied(rows_scale=1 / 32)
    res = run_fakequant("nvfp4", wl["tensors"], wl["groups"], 2)
    am = oracle.tied_amax(wl["tensors"], wl["groups"], 2)
    assert_same("tied amax", res["amax"].view(np.uint32), am.view(np.uint32))
    st = np.array([oracle.nvfp4_tensor_scale(a) for a in am], np.float32)
    assert_same("tied s_t", res["s_t"].view(np.uint32), st.view(np.uint32))
    compare_full("nvfp4", wl["tensors"], res, am, wl["groups"], label="tied")
    # STE backward, identity and clipped, on the upstream gradients
    amax_d = torch.from_numpy(am).to(DEV)
    for i, (x, g) in enumerate(zip(wl["tensors"], wl["grads"])):
        gd, xd = g.to(DEV), x.to(DEV)
        out = torch.empty_like(gd)
        qf.qf_ste_backward(gd, out, mode=0)
        torch.cuda.synchronize()
        assert_same(f"ste identity {i}", bits(out), oracle.ste_backward(g))
        qf.qf_ste_backward(gd, out, mode=1, fmt="nvfp4", x=xd, group=wl["groups"][i],
                           group_amax=amax_d)
        torch.cuda.synchronize()
        want = oracle.ste_backward(g, 1, "nvfp4", x, am[wl["groups"][i]])
        assert_same(f"ste clipped {i}", bits(out), want)


@pytest.mark.parametrize("fmt", ["mxfp4", "q4k"])
def test_ste_clipped_other_formats(fmt):
    x = workloads.nvfp4_tied(rows_scale=1 / 64)["tensors"][1]
    g = workloads.normal_with_outliers(x.shape[0], x.shape[1], 1e-3, 0, 1, 3, 77)
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=DEV)
    qf.qf_ste_backward(g.to(DEV), out, mode=1, fmt=fmt, x=x.to(DEV))
    torch.cuda.synchronize()
    assert_same(f"ste clipped {fmt}", bits(out), oracle.ste_backward(g, 1, fmt, x))


def test_activation_tracked_amax():
    """NVFP4 activation fake-quant with the running amax: tracked = max(tracked, amax)
    and the tensor scale comes from the tracked value."""
    a = workloads.nvfp4_activation(rows_scale=1 / 256)["tensors"][0]
    am = oracle.amax(a)
    for start in (0.0, 2.0 * am, 0.5 * am):
        res = run_fakequant("nvfp4", [a], tracked=[start])
        want_tr = np.float32(max(np.float32(start), np.float32(am)))
        assert_same("tracked", res["tracked"].view(np.uint32), np.array([want_tr]).view(np.uint32))
        assert_same("cur amax", res["amax"].view(np.uint32), np.float32([am]).view(np.uint32))
        compare_full("nvfp4", [a], res, np.array([want_tr]), label="act")


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_pack_equals_fakequant_codes(fmt):
    wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False)
    full = run_fakequant(fmt, wl["tensors"], wl["groups"], 2)
    pk = run_fakequant(fmt, wl["tensors"], wl["groups"], 2, pack_only=True)
    for i in range(len(wl["tensors"])):
        assert pk["y"][i] is None
        assert_same(f"pack codes {i}", pk["codes"][i], full["codes"][i])
        if full["scales"][i] is not None:
            assert_same(f"pack scales {i}", pk["scales"][i], full["scales"][i])


# ----------------------------------------------------------------------------- grouped launch
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_moe_grouped_equals_looped_and_oracle(fmt):
    wl = workloads.moe_experts(n_experts=12)
    ts, groups, ng = wl["tensors"], wl["groups"], wl["n_groups"]
    grouped = run_fakequant(fmt, ts, groups, ng)
    am = oracle.tied_amax(ts, groups, ng) if fmt == "nvfp4" else None
    if fmt == "nvfp4":
        assert_same("moe amax", grouped["amax"].view(np.uint32), am.view(np.uint32))
    # each expert in its own call: the call sees only that expert's tensors
    for e in range(12):
        idx = [3 * e, 3 * e + 1, 3 * e + 2]
        sub = [ts[i] for i in idx]
        if fmt == "nvfp4":
            g_local = [0, 0, 1]
            one = run_fakequant(fmt, sub, g_local, 2)
        else:
            one = run_fakequant(fmt, sub)
        for k, i in enumerate(idx):
            assert_same(f"expert {e} y", one["y"][k], grouped["y"][i])
            assert_same(f"expert {e} codes", one["codes"][k], grouped["codes"][i])
            if one["scales"][k] is not None:
                assert_same(f"expert {e} scales", one["scales"][k], grouped["scales"][i])
    compare_full(fmt, ts[:6], {k: v[:6] for k, v in grouped.items() if isinstance(v, list)},
                 am, groups[:6], label=f"moe {fmt}")


def test_more_tensors_than_one_descriptor_table():
    """A call with more tensors than one launch's descriptor table holds."""
    rng_shapes = [(1 + (i % 5), 32 * (1 + (i % 7))) for i in range(451)]
    ts = [workloads.normal_with_outliers(r, c, 0.02, 1e-2, 20, 8, i) for i, (r, c) in
          enumerate(rng_shapes)]
    groups = [i % 37 for i in range(len(ts))]
    for fmt in ("nvfp4", "mxfp4"):
        res = run_fakequant(fmt, ts, groups, 37)
        am = oracle.tied_amax(ts, groups, 37) if fmt == "nvfp4" else None
        compare_full(fmt, ts, res, am, groups, label=f"many {fmt}")


# ----------------------------------------------------------------------------- edge cases
def _edge_tensors():
    out = []
    z = torch.zeros(2, 256, dtype=torch.bfloat16)
    z.view(torch.int16)[0, 5] = -32768                 # a negative zero
    out.append(("zeros", z))
    tiny = torch.full((1, 256), 0, dtype=torch.int16)
    tiny[0, ::3] = 1
    tiny[0, 1::3] = -32768 | 3
    out.append(("subnormal", tiny.view(torch.bfloat16)))
    big = workloads.normal_with_outliers(3, 512, 1e37, 0.0, 1.0, 5, 0)
    big.view(torch.int16)[1, 7] = 0x7F7F                 # largest finite BF16
    out.append(("huge", big))
    one = workloads.normal_with_outliers(1, 256, 1.0, 0.0, 1.0, 6, 0)
    out.append(("one_superblock", one))
    ragged = workloads.normal_with_outliers(3, 768, 0.02, 1e-2, 20.0, 7, 0)   # 2304 elements
    out.append(("ragged", ragged))
    pos = workloads.normal_with_outliers(5, 256, 0.02, 0.0, 1.0, 9, 0).abs() + 0.001
    out.append(("positive", pos.to(torch.bfloat16)))
    # values just above the smallest normal (BF16 bit patterns 0x0080..0x00BF, mixed signs):
    # a sub-block's range is below 18 * 2^-128, so its trial scales' reciprocals overflow
    # (the MSE search's 0 * inf case); row 0 holds such a sub-block inside a normal
    # super-block
    g = torch.Generator().manual_seed(11)
    lo = torch.randint(0x0080, 0x00C0, (2, 256), generator=g, dtype=torch.int32)
    lo = torch.where(torch.rand(2, 256, generator=g) < 0.5, lo, lo | 0x8000).to(torch.int16)
    mixed = workloads.normal_with_outliers(2, 256, 0.02, 0.0, 1.0, 12, 0)
    mixed.view(torch.int16)[0, 32:64] = lo[0, 32:64]
    out.append(("near_min_normal_in_normal", mixed))
    out.append(("near_min_normal", lo.view(torch.bfloat16).contiguous()))
    return out


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k", "q4k_mse"])
def test_edge_cases_each_alone(fmt):
    for name, x in _edge_tensors():
        if fmt in ("q4k", "q4k_mse") and name == "huge":
            continue        # beyond what Q4_K's FP16 super-block scale can hold
        res = run_fakequant(fmt, [x])
        am = oracle.tied_amax([x], [0], 1) if fmt == "nvfp4" else None
        compare_full(fmt, [x], res, am, label=f"{fmt} {name}")


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_small_ragged_shapes(fmt):
    blk = 16 if fmt == "nvfp4" else 32
    shapes = [(1, blk), (3, blk), (1, 3 * blk), (7, 5 * blk), (2, 1024 + blk), (33, 2 * blk)]
    ts = [workloads.normal_with_outliers(r, c, 0.02, 5e-2, 20.0, 10, i) for i, (r, c) in
          enumerate(shapes)]
    res = run_fakequant(fmt, ts, list(range(len(ts))), len(ts))
    am = oracle.tied_amax(ts, list(range(len(ts))), len(ts)) if fmt == "nvfp4" else None
    compare_full(fmt, ts, res, am, list(range(len(ts))), label=f"{fmt} ragged")


def test_nvfp4_reciprocal_overflow_block():
    x = torch.zeros(1, 16, dtype=torch.int16)
    x[0, 0] = 1
    x[0, 1] = -32768
    x[0, 2] = -32768 | 1
    xb = x.view(torch.bfloat16)
    res = run_fakequant("nvfp4", [xb])
    am = oracle.tied_amax([xb], [0], 1)
    compare_full("nvfp4", [xb], res, am, label="rcp overflow")


def test_empty_tensors_and_calls():
    x = torch.zeros(0, 4096, dtype=torch.bfloat16, device=DEV)
    amax = torch.full((2,), 7.0, device=DEV)
    qf.qf_amax_tied([x], [1], amax)
    torch.cuda.synchronize()
    assert amax.tolist() == [0.0, 0.0]
    y = torch.empty_like(x)
    c = torch.empty(0, dtype=torch.uint8, device=DEV)
    for fmt in ("mxfp4", "q4k"):
        qf.qf_fakequant(fmt, [x], [y], [c], [c])
        qf.qf_fakequant(fmt, [])
    so = torch.full((2,), float("nan"), device=DEV)
    qf.qf_fakequant("nvfp4", [x], [y], [c], [c], groups=[0], group_amax=amax, group_scale_out=so)
    torch.cuda.synchronize()
    assert so.tolist() == [0.0, 0.0]


def test_amax_ragged_element_counts():
    """qf_amax_tied accepts any cols; tails shorter than 8 elements are included."""
    ts = [workloads.normal_with_outliers(r, c, 1.0, 0.0, 1.0, 12, i)
          for i, (r, c) in enumerate([(1, 3), (3, 5), (2, 1031), (1, 1)])]
    ts[1].view(torch.int16)[2, 4] = 0x4700                 # 32768: the max, in the last element
    xs = [t.to(DEV) for t in ts]
    amax = torch.empty(2, device=DEV)
    qf.qf_amax_tied(xs, [0, 1, 0, 1], amax)
    torch.cuda.synchronize()
    want = oracle.tied_amax(ts, [0, 1, 0, 1], 2)
    assert_same("ragged amax", amax.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_errors_launch_nothing():
    x = torch.zeros(4, 48, dtype=torch.bfloat16, device=DEV)
    y = torch.full_like(x, 3.0)
    c = torch.zeros(96, dtype=torch.uint8, device=DEV)
    with pytest.raises(qf.QfError) as ei:
        qf.qf_fakequant("mxfp4", [x], [y], [c], [c])          # 48 is not a multiple of 32
    assert ei.value.status == 2
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
    with pytest.raises(qf.QfError) as ei:
        qf.qf_fakequant("nvfp4", [x], [y], [c], [c], groups=[3],
                        group_amax=torch.ones(2, device=DEV))
    assert ei.value.status == 1
    buf = torch.zeros(4 * 32 + 1, dtype=torch.bfloat16, device=DEV)
    xm = buf[1:].view(4, 32)                                # 2 bytes past a 16-byte boundary
    with pytest.raises(qf.QfError) as ei:
        qf.qf_fakequant("mxfp4", [xm], [y[:, :32].contiguous()], [c], [c])
    assert ei.value.status == 3


# ----------------------------------------------------------------------------- full sizes
@pytest.mark.slow
def test_full_nvfp4_weight_whole():
    wl = workloads.nvfp4_weight()
    res = run_fakequant("nvfp4", wl["tensors"])
    am = oracle.tied_amax(wl["tensors"], [0], 1)
    compare_full("nvfp4", wl["tensors"], res, am, label="w4096")


# The other full-size configurations are compared whole, every output byte, in
# tests/test_gpu_fullsize.py.


# ----------------------------------------------------------------------------- FP32 latent input
def _f32_weights(rows, cols, seed, std=0.02, outliers=1e-3):
    rng = np.random.default_rng([seed, 7])
    a = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    k = int(round(outliers * a.size))
    if k:
        idx = rng.choice(a.size, size=k, replace=False)
        a.reshape(-1)[idx] *= np.float32(20.0)
    return torch.from_numpy(a)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_f32_latent_weights(fmt):
    """FP32 master weights (not BF16-representable) through every format, grouped."""
    shapes = [(64, 4096), (16, 4096), (16, 4096), (48, 1024), (3, 256)]
    ts = [_f32_weights(r, c, 60 + i) for i, (r, c) in enumerate(shapes)]
    groups = [0, 0, 0, 1, 1]
    res = run_fakequant(fmt, ts, groups, 2)
    am = oracle.tied_amax(ts, groups, 2) if fmt == "nvfp4" else None
    if fmt == "nvfp4":
        assert_same("f32 amax", res["amax"].view(np.uint32), am.view(np.uint32))
    compare_full(fmt, ts, res, am, groups, label=f"f32 {fmt}")


def test_f32_equal_to_bf16_when_representable():
    wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False)
    for fmt in ("nvfp4", "mxfp4", "q4k"):
        a = run_fakequant(fmt, wl["tensors"], wl["groups"], 2)
        b = run_fakequant(fmt, [t.float() for t in wl["tensors"]], wl["groups"], 2)
        for k in ("y", "codes", "scales"):
            for u, v in zip(a[k], b[k]):
                if u is not None:
                    assert_same(f"{fmt} {k}", v, u)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_f32_clipped_ste_and_ragged_amax(fmt):
    x = _f32_weights(8, 512, 70, std=0.05, outliers=2e-2)
    g = workloads.normal_with_outliers(8, 512, 1e-3, 0, 1, 3, 71)
    am = oracle.tied_amax([x], [0], 1)
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=DEV)
    qf.qf_ste_backward(g.to(DEV), out, mode=1, fmt=fmt, x=x.to(DEV), group=0,
                       group_amax=torch.from_numpy(am).to(DEV) if fmt == "nvfp4" else None)
    torch.cuda.synchronize()
    assert_same(f"f32 ste {fmt}", bits(out), oracle.ste_backward(g, 1, fmt, x, float(am[0])))
    ts = [_f32_weights(r, c, 80 + i) for i, (r, c) in enumerate([(1, 3), (3, 5), (2, 1031)])]
    amax = torch.empty(1, device=DEV)
    qf.qf_amax_tied([t.to(DEV) for t in ts], [0, 0, 0], amax)
    torch.cuda.synchronize()
    want = oracle.tied_amax(ts, [0, 0, 0], 1)
    assert_same("f32 ragged amax", amax.cpu().numpy().view(np.uint32), want.view(np.uint32))


# ----------------------------------------------------------------------------- Q4_K, MSE-searched fit
def test_q4k_mse_small_and_ragged():
    wl = workloads.q4k_weights(rows_scale=1 / 64)
    ts = wl["tensors"] + [workloads.normal_with_outliers(3, 768, 0.02, 1e-2, 20.0, 7, 0),
                          _f32_weights(5, 256, 90)[:, :256].contiguous()]
    res = run_fakequant("q4k_mse", ts[:3])
    compare_full("q4k_mse", ts[:3], res, label="q4k mse")
    for i, t in enumerate(ts[3:]):                 # one element type per call
        res = run_fakequant("q4k_mse", [t])
        compare_full("q4k_mse", [t], res, label=f"q4k mse extra {i}")


def test_q4k_mse_pack_and_clipped_ste():
    x = workloads.q4k_weights(rows_scale=1 / 256)["tensors"][1]
    full = run_fakequant("q4k_mse", [x])
    pk = run_fakequant("q4k_mse", [x], pack_only=True)
    assert_same("q4k mse pack", pk["codes"][0], full["codes"][0])
    g = workloads.normal_with_outliers(x.shape[0], x.shape[1], 1e-3, 0, 1, 3, 91)
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=DEV)
    qf.qf_ste_backward(g.to(DEV), out, mode=1, fmt="q4k_mse", x=x.to(DEV))
    torch.cuda.synchronize()
    assert_same("q4k mse ste", bits(out), oracle.ste_backward(g, 1, "q4k_mse", x))


def test_q4k_clipped_ste_at_both_ends_of_the_code_range():
    """Elements that scale to exactly 0 and exactly 15 keep their gradient on the device
    too (the super-block of workloads.q4k_ste_ends)."""
    x = workloads.q4k_ste_ends()
    g = workloads.normal_with_outliers(1, 256, 1e-3, 0.0, 1.0, 52, 0)
    want = oracle.ste_backward(g, 1, "q4k", x)
    assert want.reshape(-1)[32] != 0 and want.reshape(-1)[64] != 0
    out = torch.empty(1, 256, dtype=torch.bfloat16, device=DEV)
    qf.qf_ste_backward(g.to(DEV), out, mode=1, fmt="q4k", x=x.to(DEV))
    torch.cuda.synchronize()
    assert_same("q4k clipped STE ends", bits(out), want)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "q4k"])
def test_clipped_ste_in_place(fmt):
    """Clipped STE with grad_x == grad_y gives the out-of-place result (and the oracle's)."""
    wl = workloads.nvfp4_tied(rows_scale=1 / 64)
    x = wl["tensors"][3]
    gy = wl["grads"][3]
    am = float(oracle.amax(x))
    want = oracle.ste_backward(gy, 1, fmt, x, am)
    xd, g1 = x.to(DEV), gy.to(DEV)
    amax = torch.tensor([am], device=DEV)
    out = torch.empty_like(g1)
    qf.qf_ste_backward(g1, out, 1, fmt, xd, 0, amax)
    g2 = gy.to(DEV)
    qf.qf_ste_backward(g2, g2, 1, fmt, xd, 0, amax)               # in place
    torch.cuda.synchronize()
    assert_same(f"{fmt} clipped STE", bits(out), want)
    assert_same(f"{fmt} clipped STE in place", bits(g2), want)
