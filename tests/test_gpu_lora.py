"""GPU parity of the LoRA-merged fake-quant (bit for bit against the oracle).

LoRA-QAD (QATFactory project page, Method, "QAD") quantizes W + scale * B A.  The
fused calls form the BF16 merged weight on the fly; they must equal the oracle's
merge followed by its quantizer, and the library's own merge followed by
qf_fakequant."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import oracle
import workloads
from gpu_helpers import DEV, assert_same, bits, u8

pytestmark = pytest.mark.gpu


def _case(rows, cols, rank, seed):
    w = workloads.normal_with_outliers(rows, cols, 0.02, 1e-3, 20.0, seed, 0)
    b = workloads.normal_with_outliers(rows, rank, 0.01, 0.0, 1.0, seed, 1)
    a = workloads.normal_with_outliers(rank, cols, 0.02, 0.0, 1.0, seed, 2)
    return w, b, a


# Whole 64-row tiles take a guard-free path and ragged ones the guarded path; the merge
# and amax modes bring W through a 4-step ring at rank <= 16 and a 3-step ring at rank
# 32.  (130, 1040, 16), (200, 1536, 12) and (128, 2048, 32) mix whole tiles, a ragged
# row tail and a partial 1024-column group in one tensor.
SHAPES = [(37, 1040, 3), (64, 2048, 8), (33, 768, 16), (40, 4096, 32), (1, 32, 1),
          (130, 1040, 16), (200, 1536, 12), (128, 2048, 32)]


@pytest.mark.parametrize("rows,cols,rank", SHAPES)
def test_lora_merge_and_amax(rows, cols, rank):
    w, b, a = _case(rows, cols, rank, rows + rank)
    scale = 32.0 / rank
    want = oracle.lora_merge(w, b, a, scale)
    m = torch.empty(rows, cols, dtype=torch.bfloat16, device=DEV)
    adapters = [(b.to(DEV), a.to(DEV), scale)]
    qf.qf_lora_merge([w.to(DEV)], adapters, [m])
    amax = torch.empty(1, device=DEV)
    qf.qf_amax_tied_lora([w.to(DEV)], adapters, [0], amax)
    torch.cuda.synchronize()
    assert_same("merged", bits(m), want)
    assert_same("merged amax", amax.cpu().numpy().view(np.uint32),
                np.float32([oracle.amax(want)]).view(np.uint32))


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("rows,cols,rank", SHAPES)
def test_lora_fakequant_equals_merge_then_quantize(fmt, rows, cols, rank):
    if fmt == "mxfp4" and cols % 32:
        pytest.skip("MXFP4 needs 32 | cols")
    w, b, a = _case(rows, cols, rank, 3 * rows + rank)
    scale = 16.0 / rank
    merged = oracle.lora_merge(w, b, a, scale)
    am = oracle.amax(merged)
    if fmt == "nvfp4":
        y, c, s, _ = oracle.nvfp4(merged, am)
    else:
        y, c, s = oracle.mxfp4(merged)
    wd = w.to(DEV)
    adapters = [(b.to(DEV), a.to(DEV), scale)]
    yo, co, so = qf.alloc_outputs(fmt, wd)
    amax = torch.empty(1, device=DEV)
    kw = {}
    if fmt == "nvfp4":
        qf.qf_amax_tied_lora([wd], adapters, [0], amax)
        kw = {"groups": [0], "group_amax": amax}
    qf.qf_fakequant_lora(fmt, [wd], adapters, [yo], [co], [so], **kw)
    torch.cuda.synchronize()
    assert_same("lora y", bits(yo), y)
    assert_same("lora codes", u8(co), c)
    assert_same("lora scales", u8(so), s)
    # the library's own merge followed by qf_fakequant gives the same bytes
    m = torch.empty_like(wd)
    qf.qf_lora_merge([wd], adapters, [m])
    y2, c2, s2 = qf.alloc_outputs(fmt, wd)
    qf.qf_fakequant(fmt, [m], [y2], [c2], [s2], **kw)
    torch.cuda.synchronize()
    assert torch.equal(y2, yo) and torch.equal(c2, co) and torch.equal(s2, so)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_lora_fakequant_near_min_normal(fmt):
    """Merged weights just above the smallest normal (BF16 bit patterns 0x0080..0x00BF):
    an MXFP4 block there takes scale byte 0 (2^-127) with nonzero codes."""
    g = torch.Generator().manual_seed(21)
    bits16 = torch.randint(0x0080, 0x00C0, (4, 256), generator=g, dtype=torch.int32)
    bits16 = torch.where(torch.rand(4, 256, generator=g) < 0.5, bits16, bits16 | 0x8000)
    w = bits16.to(torch.int16).view(torch.bfloat16).contiguous()
    b = torch.zeros(4, 2, dtype=torch.bfloat16)
    a = torch.zeros(2, 256, dtype=torch.bfloat16)
    merged = oracle.lora_merge(w, b, a, 1.0)
    if fmt == "nvfp4":
        y, c, s, _ = oracle.nvfp4(merged, oracle.amax(merged))
    else:
        y, c, s = oracle.mxfp4(merged)
    wd = w.to(DEV)
    yo, co, so = qf.alloc_outputs(fmt, wd)
    amax = torch.empty(1, device=DEV)
    adapters = [(b.to(DEV), a.to(DEV), 1.0)]
    if fmt == "nvfp4":
        qf.qf_amax_fakequant_lora([wd], adapters, [yo], [co], [so], [0], amax)
    else:
        qf.qf_fakequant_lora(fmt, [wd], adapters, [yo], [co], [so])
    torch.cuda.synchronize()
    assert_same(f"lora {fmt} near-min y", bits(yo), y)
    assert_same(f"lora {fmt} near-min codes", u8(co), c)
    assert_same(f"lora {fmt} near-min scales", u8(so), s)


def test_lora_grouped_experts_with_tied_groups():
    """Several adapted tensors in one launch (gate/up tied, down its own group)."""
    ts, ads, groups, merged = [], [], [], []
    for e in range(3):
        for j, (r, c) in enumerate([(96, 2048), (96, 2048), (256, 768)]):
            w, b, a = _case(r, c, 16, 100 + 3 * e + j)
            ts.append(w)
            ads.append((b, a, 2.0))
            groups.append(2 * e + (j == 2))
            merged.append(oracle.lora_merge(w, b, a, 2.0))
    am = np.zeros(6, np.float32)
    for m, g in zip(merged, groups):
        am[g] = max(am[g], np.float32(oracle.amax(m)))
    xs = [t.to(DEV) for t in ts]
    adapters = [(b.to(DEV), a.to(DEV), s) for b, a, s in ads]
    amax = torch.empty(6, device=DEV)
    qf.qf_amax_tied_lora(xs, adapters, groups, amax)
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    so = torch.empty(6, device=DEV)
    qf.qf_fakequant_lora("nvfp4", xs, adapters, [o[0] for o in outs], [o[1] for o in outs],
                         [o[2] for o in outs], groups, amax, so)
    torch.cuda.synchronize()
    assert_same("grouped lora amax", amax.cpu().numpy().view(np.uint32), am.view(np.uint32))
    for i, m in enumerate(merged):
        y, c, s, _ = oracle.nvfp4(m, am[groups[i]])
        assert_same(f"grouped lora y {i}", bits(outs[i][0]), y)
        assert_same(f"grouped lora codes {i}", u8(outs[i][1]), c)
        assert_same(f"grouped lora scales {i}", u8(outs[i][2]), s)


@pytest.mark.parametrize("rows,cols,rank", SHAPES)
@pytest.mark.parametrize("with_y", [True, False])
def test_amax_fakequant_lora_one_call(rows, cols, rank, with_y):
    """qf_amax_fakequant_lora: with y, the merged weight is formed once and quantized in
    place; without y, it is formed in both passes.  Either way the bytes are the
    oracle's (merge, then tie-group amax, then NVFP4)."""
    if cols % 16:
        pytest.skip("NVFP4 needs 16 | cols")
    w, b, a = _case(rows, cols, rank, 5 * rows + rank)
    scale = 24.0 / rank
    merged = oracle.lora_merge(w, b, a, scale)
    am = np.float32(oracle.amax(merged))
    y, c, s, st = oracle.nvfp4(merged, am)
    wd = w.to(DEV)
    yo, co, so = qf.alloc_outputs("nvfp4", wd)
    amax = torch.full((1,), float("nan"), device=DEV)
    st_out = torch.full((1,), float("nan"), device=DEV)
    qf.qf_amax_fakequant_lora([wd], [(b.to(DEV), a.to(DEV), scale)], [yo] if with_y else None,
                              [co], [so], [0], amax, st_out)
    torch.cuda.synchronize()
    assert_same("one-call amax", amax.cpu().numpy().view(np.uint32), np.float32([am]).view(np.uint32))
    assert_same("one-call s_t", st_out.cpu().numpy().view(np.uint32), np.float32([st]).view(np.uint32))
    if with_y:
        assert_same("one-call y", bits(yo), y)
    assert_same("one-call codes", u8(co), c)
    assert_same("one-call scales", u8(so), s)


def test_amax_fakequant_lora_grouped():
    """Experts with tied groups in one call, merged weights formed once."""
    ts, ads, groups, merged = [], [], [], []
    for e in range(3):
        for j, (r, c) in enumerate([(96, 2048), (96, 2048), (256, 768)]):
            w, b, a = _case(r, c, 8, 300 + 3 * e + j)
            ts.append(w)
            ads.append((b, a, 3.0))
            groups.append(2 * e + (j == 2))
            merged.append(oracle.lora_merge(w, b, a, 3.0))
    am = np.zeros(6, np.float32)
    for m, g in zip(merged, groups):
        am[g] = max(am[g], np.float32(oracle.amax(m)))
    xs = [t.to(DEV) for t in ts]
    adapters = [(b.to(DEV), a.to(DEV), s) for b, a, s in ads]
    amax = torch.empty(6, device=DEV)
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    qf.qf_amax_fakequant_lora(xs, adapters, [o[0] for o in outs], [o[1] for o in outs],
                              [o[2] for o in outs], groups, amax)
    torch.cuda.synchronize()
    assert_same("grouped one-call amax", amax.cpu().numpy().view(np.uint32), am.view(np.uint32))
    for i, m in enumerate(merged):
        y, c, s, _ = oracle.nvfp4(m, am[groups[i]])
        assert_same(f"grouped one-call y {i}", bits(outs[i][0]), y)
        assert_same(f"grouped one-call codes {i}", u8(outs[i][1]), c)
        assert_same(f"grouped one-call scales {i}", u8(outs[i][2]), s)


@pytest.mark.parametrize("rank_pad", [4, 8, 16])
def test_merge_accumulates_in_increasing_k(rank_pad):
    """The oracle pin's worked case on the device: products 1, 2^-8, 2^-24, 2^-24 in
    increasing k give BF16 1.0; in decreasing k, 1 + 2^-7.  Extra zero ranks (rank_pad)
    add exact zeros.  Every column carries the same products."""
    cols = 32
    prods = [1.0, 2.0 ** -4, 2.0 ** -12, 2.0 ** -12] + [0.0] * (rank_pad - 4)
    for order, want in ((1, 0x3F80), (-1, 0x3F81)):
        p = prods[:4][::order] + prods[4:]
        b = torch.tensor([p], dtype=torch.bfloat16, device=DEV)
        a = torch.tensor(p, dtype=torch.bfloat16, device=DEV)[:, None].repeat(1, cols).contiguous()
        w = torch.zeros(1, cols, dtype=torch.bfloat16, device=DEV)
        m = torch.empty_like(w)
        qf.qf_lora_merge([w], [(b, a, 1.0)], [m])
        torch.cuda.synchronize()
        assert np.all(bits(m) == want), (order, [hex(v) for v in bits(m)[:4]])


def test_underflowing_product_is_fused_on_the_device():
    """The oracle's worked case (products 2^-149 then 2^-150; W = 0, scale = 2^100):
    the device's fused terms give the merged weight 2^-48, as the oracle does, in the
    merge call and in the fused fake-quant."""
    cols = 32
    w = torch.zeros(1, cols, dtype=torch.bfloat16)
    b = torch.tensor([[2.0 ** -75, 2.0 ** -75]], dtype=torch.bfloat16)
    a = torch.tensor([[2.0 ** -74] * cols, [2.0 ** -75] * cols], dtype=torch.bfloat16)
    scale = 2.0 ** 100
    want = oracle.lora_merge(w, b, a, scale)
    assert int(want[0, 0]) == 0x2780
    wd = w.to(DEV)
    m = torch.empty_like(wd)
    qf.qf_lora_merge([wd], [(b.to(DEV), a.to(DEV), scale)], [m])
    torch.cuda.synchronize()
    assert_same("fused merge", bits(m), want)
    y, c, s = qf.alloc_outputs("mxfp4", wd)
    qf.qf_fakequant_lora("mxfp4", [wd], [(b.to(DEV), a.to(DEV), scale)], [y], [c], [s])
    torch.cuda.synchronize()
    yo, co, so = oracle.mxfp4(want)
    assert_same("fused merge, MXFP4 y", bits(y), yo)
    assert_same("fused merge, MXFP4 codes", u8(c), co)


# ----------------------------------------------------------------------------- merged amax
# qf_amax_tied_lora evaluates the merge only where a bound on |M| reaches a lower bound
# of the group's max; these cases make the bounds decide the result, or make them
# useless, and compare the group amax with the oracle's (merge, then max |M|).
def _amax_case(ts, ads, groups, ng):
    want = np.zeros(ng, np.float32)
    for (w, (b, a, s)), g in zip(zip(ts, ads), groups):
        want[g] = max(want[g], np.float32(oracle.amax(oracle.lora_merge(w, b, a, s))))
    amax = torch.full((ng,), float("nan"), device=DEV)
    qf.qf_amax_tied_lora([w.to(DEV) for w in ts], [(b.to(DEV), a.to(DEV), s) for b, a, s in ads],
                         groups, amax)
    torch.cuda.synchronize()
    assert_same("merged amax", amax.cpu().numpy().view(np.uint32), want.view(np.uint32))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_merged_amax_where_the_merge_moves_the_max():
    """The largest |W| shrinks and the second largest grows past it: the max is not at
    the argmax of |W|, and both lie inside each other's bounds."""
    rows, cols, r = 64, 1024, 4
    w = np.zeros((rows, cols), np.float32)
    w[5, 100], w[40, 900] = 1.0, 0.98
    b = np.zeros((rows, r), np.float32)
    a = np.zeros((r, cols), np.float32)
    b[5, 0], a[0, 100] = 0.25, -0.125                      # M[5,100] = 1 - 2 * 0.03125
    b[40, 1], a[1, 900] = 0.25, 0.125                       # M[40,900] = 0.98 + 0.0625
    _amax_case([_bf16(w)], [(_bf16(b), _bf16(a), 2.0)], [0], 1)


@pytest.mark.parametrize("case", ["zero_base", "zero_adapter", "zero_scale", "negative_scale",
                                  "huge_scale", "ties", "subnormal_base", "all_zero"])
def test_merged_amax_edge_cases(case):
    rows, cols, r = 70, 1040, 8                            # a ragged row tile and column group
    w = workloads.normal_with_outliers(rows, cols, 0.02, 1e-3, 20.0, 31, 0)
    b = workloads.normal_with_outliers(rows, r, 0.01, 0.0, 1.0, 31, 1)
    a = workloads.normal_with_outliers(r, cols, 0.02, 0.0, 1.0, 31, 2)
    s = 2.0
    if case == "zero_base":          # the max comes from the merge alone: no pruning possible
        w = torch.zeros_like(w)
    elif case == "zero_adapter":     # B = 0 (the usual initialisation): M = W exactly
        b = torch.zeros_like(b)
    elif case == "zero_scale":
        s = 0.0
    elif case == "negative_scale":
        s = -3.0
    elif case == "huge_scale":       # the bounds overflow to inf: every element is evaluated
        s = 1e30
    elif case == "ties":             # many elements share the largest |W|
        w = torch.where(w.abs() > 0.03, torch.sign(w) * 0.5, w).to(torch.bfloat16)
    elif case == "subnormal_base":   # BF16 subnormals with a tiny adapter
        w = (w.float() * 1e-37).to(torch.bfloat16)
        b = (b.float() * 1e-20).to(torch.bfloat16)
        a = (a.float() * 1e-19).to(torch.bfloat16)
    elif case == "all_zero":
        w, b = torch.zeros_like(w), torch.zeros_like(b)
    _amax_case([w], [(b, a, s)], [0], 1)


def test_merged_amax_many_tensors_and_groups():
    """Expert-like tensors in several tie groups, each spread over many CTAs."""
    ts, ads, groups = [], [], []
    for e in range(4):
        for j, (rr, c) in enumerate([(200, 2048), (200, 2048), (512, 768)]):
            w, b, a = _case(rr, c, 16, 700 + 3 * e + j)
            ts.append(w)
            ads.append((b, a, 2.0))
            groups.append(2 * e + (j == 2))
    _amax_case(ts, ads, groups, 8)


@pytest.mark.parametrize("case", ["pow2_1", "pow2_8", "half", "pow2_overflow_guard", "odd"])
def test_merge_paths_for_scale_kinds(case):
    """The merge rounds W + scale * acc once when scale is a power of two >= 1 and a bound
    rules out overflow, else as a rounded product and a rounded add; both must give the
    oracle's bytes.  In the guard case (adapters scaled by 1e5, scale 2^100) the bound on
    scale * acc exceeds 2^126, so the two-rounding path must run, while the values stay
    finite (about 5e37 at most)."""
    rows, cols, r = 130, 2048, 16
    w, b, a = _case(rows, cols, r, 900)
    scale = {"pow2_1": 1.0, "pow2_8": 8.0, "half": 0.5, "pow2_overflow_guard": 2.0 ** 100,
             "odd": 3.0}[case]
    if case == "pow2_overflow_guard":
        b = (b.float() * 1e5).to(torch.bfloat16)
        a = (a.float() * 1e5).to(torch.bfloat16)
    merged = oracle.lora_merge(w, b, a, scale)
    wd = w.to(DEV)
    ad = [(b.to(DEV), a.to(DEV), scale)]
    m = torch.empty_like(wd)
    qf.qf_lora_merge([wd], ad, [m])
    yo, co, so = qf.alloc_outputs("nvfp4", wd)
    amax = torch.empty(1, device=DEV)
    qf.qf_amax_fakequant_lora([wd], ad, [yo], [co], [so], [0], amax)
    torch.cuda.synchronize()
    assert np.isfinite(oracle.bf16_to_f32(merged)).all()
    assert_same(f"{case} merge", bits(m), merged)
    am = np.float32(oracle.amax(merged))
    assert_same(f"{case} amax", amax.cpu().numpy().view(np.uint32), np.float32([am]).view(np.uint32))
    y, c, s, _ = oracle.nvfp4(merged, am)
    assert_same(f"{case} y", bits(yo), y)
    assert_same(f"{case} codes", u8(co), c)
