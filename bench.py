#!/usr/bin/env python3
"""Benchmark of the fused fake-quant + pack pass on B200.

Default (headline) workload `w4a4`: MXFP4 W4A4 -- weight BF16 12288x4096
N(0, 0.02) and activations 8 x 4096 tokens by 4096 hidden, Student-t(3) with 1%
of channels x50 -- quantized in ONE grouped qf_fakequant launch that writes
dequantized BF16, packed E2M1 nibbles and E8M0 block scales.  A step is that
launch.  Other workloads (`--workload`): nvfp4_tied, q4k, nvfp4_weight,
activation, moe_nvfp4, moe_mxfp4, moe_q4k, nvfp4_tied_f32, q4k_f32 (FP32 master
weights), lora_nvfp4 (LoRA-merged weights), lora_amax (their tie-group amax alone),
q4k_mse (MSE-searched Q4_K fit); an NVFP4 step is the tied-amax pass followed by the
fused pass.

  value      GB/s of algorithmic bytes per step (read BF16 + write BF16 + codes +
             scales = 4.5625 / 4.53125 / 4.5625 B per element for NVFP4 / MXFP4 /
             Q4_K, plus 2 B per element for an NVFP4 amax pass), device-timed,
             max over ranks, summed over ranks (weak scaling).
  e2e        the same metric through the public API with pinned host buffers:
             host->device copy of the inputs, the step, device->host copy of every
             output, per step, pipelined in row chunks (host.HostPipeline).
  roofline   the fused-pass kernel's achieved GB/s (its algorithmic bytes / its
             mean CUDA-event duration in the timed region) against the measured
             HBM copy bandwidth.
  cpu_baseline  the oracle (scalar C) on a bounded sample of the rows, on every host core
             of the affinity mask (rows split over threads), plus a one-core figure.
  pack_only  the same launch writing codes and scales only (no BF16 dequant): the
             input read plus 0.5625 / 0.53125 / 0.5625 B per element.
  per_format the other workloads, each timed per call with the L2 flushed
             (L2Flush: L2 left holding only clean lines), with their pack-only launch.
  per_format_summary  the line's last key: compact figures for every workload.

`--impl reference` times the oracle on the host cores for the same metric (the
reference arm).  Launch with torchrun for N > 1 GPUs (one process per GPU).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fake-quant+pack GB/s and Gelem/s per format; % of B200 HBM roofline"
UNIT = "GB/s"
BYTES_PER_ELEM = {"nvfp4": 2 + 2 + 0.5 + 1 / 16, "mxfp4": 2 + 2 + 0.5 + 1 / 32,
                  "q4k": 2 + 2 + 144 / 256, "q4k_mse": 2 + 2 + 144 / 256}
# pack only (codes and scales, no BF16 dequant): output bytes per element beside the input
PACK_BYTES = {"nvfp4": 0.5 + 1 / 16, "mxfp4": 0.5 + 1 / 32, "q4k": 144 / 256}
WORKLOADS = ("w4a4", "nvfp4_tied", "q4k", "nvfp4_weight", "activation", "moe_nvfp4",
             "moe_mxfp4", "moe_q4k", "nvfp4_tied_f32", "q4k_f32", "lora_nvfp4", "lora_amax",
             "q4k_mse")


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# The MSE-searched Q4_K fit is bound by FP32 arithmetic, not by HBM.  Its algorithmic
# work per element: x + min once; for each of the nine trial scales the scaled value,
# the clamp to [0, 15] (two operations), the rounding, s*q - min (two), x - dq and the
# squared-error update (two), 9 operations; the sub-block min/max scan (two); the final
# quantize-dequantize (x + mm, the product, clamp, rounding, s*q - mm) and the BF16
# rounding (eight).  Each counts as one lane-slot of the FP32 pipe; per-sub-block work
# (the trial divides, the 6-bit scale fit) is left out.
MSE_OPS_PER_ELEM = 1 + 9 * 9 + 2 + 8
FP32_LANES_PER_SM = 128                       # 4 SM sub-partitions x 32 FP32 lanes


def fp32_peak_tops(dev, sm_max_mhz) -> tuple:
    """FP32 pipe peak in tera-operations/s: SMs x 128 lanes x the maximum SM clock."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz, src = (float(sm_max_mhz), "NVML max SM clock") if sm_max_mhz else (1965.0, "1965 MHz")
    return sms * FP32_LANES_PER_SM * mhz * 1e6 / 1e12, f"{sms} SMs x 128 FP32 lanes x {src}"


class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML (read only)."""

    REASONS = {"applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
               "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.matched = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h, self.matched = self._handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    @staticmethod
    def _handle(pynvml, index: int):
        """The NVML handle of CUDA device `index`.  NVML numbers every GPU of the machine
        while CUDA numbers the visible ones (CUDA_VISIBLE_DEVICES), so the device is
        found by its UUID; the index is the fallback."""
        try:
            u = str(torch.cuda.get_device_properties(index).uuid)
            u = u if u.startswith("GPU-") else "GPU-" + u
            return pynvml.nvmlDeviceGetHandleByUUID(u.encode()), "uuid"
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(index), "index"

    def sample_once(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.reasons |= {k for k, v in self.REASONS.items() if mask & v}
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample_once()
            time.sleep(0.002)

    def __enter__(self):
        self.sample_once()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "device_by": self.matched}


def csrc_digest() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "fp4_fake_quant_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this
    exact kernel source and workload; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        e = json.load(open(p)).get(f"{kernel}@{workload}")
        if e and e.get("csrc_sha") == csrc_digest():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def max_over_ranks(vals, device):
    """Element-wise max over all ranks (device timings are reported as the slowest rank)."""
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_value(step_bytes: float, world: int, ms_per_step: float) -> float:
    """Whole-job GB/s: every rank processes its own step of `step_bytes` per slowest step."""
    return world * step_bytes / (ms_per_step * 1e-3) / 1e9


# ----------------------------------------------------------------------------- workloads
_CACHE = {}


def make_workload(name: str, qf, dev, seed_shift: int = 0):
    """Inputs resident on `dev`, outputs allocated, and the two parts of a step:
    `pre` (the NVFP4 tied-amax pass, or None) and `fq` (the fused pass)."""
    if name == "w4a4":
        wl, fmt = workloads.mxfp4_w4a4(seed=1 + seed_shift), "mxfp4"
        desc = ("MXFP4 W4A4: weight BF16 12288x4096 N(0,0.02) + activations BF16 32768x4096 "
                "(8x4096 tokens) Student-t(3), 1% channels x50; one grouped fake-quant+pack launch")
    elif name == "nvfp4_tied":
        wl, fmt = workloads.nvfp4_tied(seed=3 + seed_shift, with_grads=False), "nvfp4"
        desc = ("NVFP4 tied fused projections: Q 4096x4096, K/V 1024x4096 (one tensor scale), "
                "gate/up 14336x4096 (another); tied amax pass + one grouped fake-quant+pack launch")
    elif name == "q4k":
        wl, fmt = workloads.q4k_weights(seed=2 + seed_shift), "q4k"
        desc = ("Q4_K weight-only: down 4096x14336 + up 14336x4096, N(0,0.015) x per-row "
                "log-uniform[0.5,2]; one grouped fake-quant+pack launch (144-byte blocks)")
    elif name == "q4k_mse":
        wl, fmt = workloads.q4k_weights(seed=2 + seed_shift), "q4k_mse"
        desc = ("Q4_K with the MSE-searched scale fit (9 trial scales per sub-block): down "
                "4096x14336 + up 14336x4096; one grouped launch (the PTQ-baseline quantizer)")
    elif name == "q4k_f32":
        wl, fmt = workloads.q4k_weights(seed=2 + seed_shift, dtype="f32"), "q4k"
        desc = ("Q4_K from FP32 latent weights: down 4096x14336 + up 14336x4096; one grouped "
                "fake-quant+pack launch (FP32 in, BF16 + 144-byte blocks out)")
    elif name == "nvfp4_tied_f32":
        wl, fmt = workloads.nvfp4_tied(seed=3 + seed_shift, with_grads=False, dtype="f32"), "nvfp4"
        desc = ("NVFP4 tied projections from FP32 latent weights (Q/K/V, gate/up); tied amax "
                "pass + one grouped fake-quant+pack launch (FP32 in, BF16 + codes out)")
    elif name == "nvfp4_weight":
        wl, fmt = workloads.nvfp4_weight(seed=0 + seed_shift), "nvfp4"
        desc = ("NVFP4 weight 4096x4096 N(0,0.02), 0.1% x20 outliers; qf_amax_fakequant: amax, "
                "grid barrier and fake-quant+pack in one cooperative launch (input L2-resident "
                "for the second pass)")
    elif name in ("moe_nvfp4", "moe_mxfp4", "moe_q4k"):
        key = ("moe", seed_shift)                    # the three formats share one input set
        if key not in _CACHE:
            _CACHE.clear()
            _CACHE[key] = workloads.moe_experts(seed=4 + seed_shift)
        wl, fmt = _CACHE[key], name[4:]
        desc = (f"MoE 128 experts x (gate, up 768x2048, down 2048x768), {fmt.upper()}; one grouped "
                "launch over 384 tensors" + (" after a tied amax pass" if fmt == "nvfp4" else ""))
    elif name == "lora_nvfp4":
        wl, fmt = workloads.nvfp4_tied(seed=3 + seed_shift, with_grads=False), "nvfp4"
        desc = ("LoRA-QAD NVFP4: tied Q/K/V and gate/up bases with rank-16 adapters (scale 2); "
                "qf_amax_fakequant_lora: the merged weight formed once (written to y with its "
                "group amax), then fake-quant+pack of y in place")
    elif name == "lora_amax":
        wl, fmt = workloads.nvfp4_tied(seed=3 + seed_shift, with_grads=False), "nvfp4"
        desc = ("LoRA-QAD NVFP4 tie-group amax of the merged weights (qf_amax_tied_lora): tied "
                "Q/K/V and gate/up bases with rank-16 adapters (scale 2), W read once, the merge "
                "evaluated exactly only where a bound reaches the group's max")
    elif name == "activation":
        wl, fmt = workloads.nvfp4_activation(seed=5 + seed_shift), "nvfp4"
        desc = ("NVFP4 activation 32768x4096 Student-t(3) with tracked amax: amax pass "
                "(running max) + fake-quant+pack")
    else:
        raise SystemExit(f"unknown workload {name}; choose from {', '.join(WORKLOADS)}")
    xs_h = [t.pin_memory() for t in wl["tensors"]]
    xs = [t.to(dev, non_blocking=True) for t in xs_h]
    groups, ng = wl["groups"], wl["n_groups"]
    outs = [qf.alloc_outputs(fmt, x) for x in xs]
    Y, C, S = [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs]
    numel = sum(x.numel() for x in xs)
    in_b = xs[0].element_size()                      # 2 (BF16) or 4 (FP32 latent weights)
    chunks = (len(xs) + 383) // 384                  # launches per call (descriptor tables)
    W = dict(name=name, fmt=fmt, desc=desc, xs=xs, xs_h=xs_h, outs=[t for t in Y + C + S if
             t is not None], numel=numel, fq_bytes=numel * (BYTES_PER_ELEM[fmt] + in_b - 2),
             n_tensors=len(xs), in_bytes=in_b, groups=groups, n_groups=ng)
    if name == "lora_amax":
        r = 16
        ads = [(workloads.normal_with_outliers(x.shape[0], r, 0.01, 0, 1, 9 + seed_shift, 2 * i)
                .to(dev), workloads.normal_with_outliers(r, x.shape[1], 0.02, 0, 1, 9 + seed_shift,
                                                         2 * i + 1).to(dev), 2.0)
               for i, x in enumerate(xs)]
        amax = torch.zeros(ng, dtype=torch.float32, device=dev)
        W["pre"] = None
        W["fq"] = qf.prepare_amax_tied_lora(xs, ads, groups, amax)
        W["fq_bytes"] = W["step_bytes"] = 2 * numel          # W read once
        W["launches"] = 1
        W["kernel"] = "k_lora_amax"
        W["adapters"] = ads
        return W
    if name == "lora_nvfp4":
        r = 16
        ads = [(workloads.normal_with_outliers(x.shape[0], r, 0.01, 0, 1, 9 + seed_shift, 2 * i)
                .to(dev), workloads.normal_with_outliers(r, x.shape[1], 0.02, 0, 1, 9 + seed_shift,
                                                         2 * i + 1).to(dev), 2.0)
               for i, x in enumerate(xs)]
        amax = torch.zeros(ng, dtype=torch.float32, device=dev)
        so = torch.empty(ng, dtype=torch.float32, device=dev)
        pre2 = qf.prepare_amax_tied_lora(xs, ads, groups, amax)
        fq2 = qf.prepare_fakequant_lora(fmt, xs, ads, Y, C, S, groups, amax, so)
        W["pre"] = None
        W["fq"] = qf.prepare_amax_fakequant_lora(xs, ads, Y, C, S, groups, amax, so)
        # algorithmic bytes of the step: the amax read of W and the fused pass; forming
        # the merged weight once costs 4 B per element more traffic (write M, read M back)
        W["step_bytes"] = W["fq_bytes"] + 2 * numel
        W["parts"] = (pre2, fq2, W["fq_bytes"])
        W["fq_bytes"] = W["step_bytes"]
        W["two_call"] = lambda: (pre2(), fq2())
        W["launches"] = 2
        W["kernel"] = "k_lora8+k_nv"
        W["adapters"] = ads
        return W
    if name == "nvfp4_weight":
        amax = torch.zeros(ng, dtype=torch.float32, device=dev)
        so = torch.empty(ng, dtype=torch.float32, device=dev)
        W["workspace"] = qf.alloc_workspace(ng, dev)
        W["pre"] = None
        W["fq"] = qf.prepare_amax_fakequant(xs, Y, C, S, groups, amax, group_scale_out=so,
                                            workspace=W["workspace"])
        W["fq_bytes"] = W["step_bytes"] = W["fq_bytes"] + in_b * numel
        W["launches"] = 1
        W["kernel"] = "k_nv_oneshot"
        # the same step as two launches (qf_amax_tied, then qf_fakequant), for comparison,
        # and its parts: the per-format table reports the fused pass alone as for the others
        pre2 = qf.prepare_amax_tied(xs, groups, amax)
        fq2 = qf.prepare_fakequant(fmt, xs, Y, C, S, groups, amax, so)
        W["two_call"] = lambda: (pre2(), fq2())
        W["parts"] = (pre2, fq2, numel * (BYTES_PER_ELEM[fmt] + in_b - 2))
        return W
    if fmt == "nvfp4":
        amax = torch.zeros(ng, dtype=torch.float32, device=dev)
        cur = torch.zeros(ng, dtype=torch.float32, device=dev)
        so = torch.empty(ng, dtype=torch.float32, device=dev)
        # prepared calls: the descriptor array is marshalled once, as a training loop would
        if name == "activation":
            W["pre"] = qf.prepare_amax_tied(xs, groups, cur, amax)     # amax <- max(amax, cur)
            W["one_call"] = qf.prepare_amax_fakequant(xs, Y, C, S, groups, cur, tracked=amax,
                                                      group_scale_out=so)
        else:
            W["pre"] = qf.prepare_amax_tied(xs, groups, amax)
            W["one_call"] = qf.prepare_amax_fakequant(xs, Y, C, S, groups, amax, group_scale_out=so)
        W["fq"] = qf.prepare_fakequant(fmt, xs, Y, C, S, groups, amax, so)
        W["pack"] = qf.prepare_fakequant(fmt, xs, None, C, S, groups, amax, so, pack_only=True)
        W["step_bytes"] = W["fq_bytes"] + in_b * numel
        W["launches"] = 2 * chunks
        W["kernel"] = "k_nv"
    else:
        W["pre"] = None
        W["fq"] = qf.prepare_fakequant(fmt, xs, Y, C, S)
        if fmt in PACK_BYTES:
            W["pack"] = qf.prepare_fakequant(fmt, xs, None, C, S, pack_only=True)
        W["step_bytes"] = W["fq_bytes"]
        W["launches"] = chunks
        W["kernel"] = {"mxfp4": "k_fp4_mxfp4", "q4k": "k_q4k", "q4k_mse": "k_q4k_mse"}[fmt]
    return W


def run_step(W):
    if W["pre"] is not None:
        W["pre"]()
    W["fq"]()


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import fp4_fake_quant_b200 as qf
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    W = make_workload(args.workload, qf, dev, seed_shift=1000 * rank)
    numel, step_bytes = W["numel"], W["step_bytes"]
    in_bytes = W["in_bytes"] * numel
    flush_buf = L2Flush(dev, l2) if in_bytes < 2 * l2 else None
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        run_step(W)
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [(E(), E(), E()) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            if flush_buf is not None:
                flush_buf()                  # L2 flush, outside the timed event pairs
            ev[i][0].record(stream)
            if W["pre"] is not None:
                W["pre"]()
            ev[i][1].record(stream)
            W["fq"]()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(c) for a, b, c in ev]
    fq_ms = [b.elapsed_time(c) for a, b, c in ev]
    total_ms = sum(step_ms) if flush_buf is not None else ev[0][0].elapsed_time(ev[-1][2])
    total_ms, kern_ms = max_over_ranks([total_ms, float(np.mean(fq_ms))], dev)
    ms_per_step = total_ms / args.steps
    value = weak_scaling_value(step_bytes, world, ms_per_step)

    # end to end through the public API with pinned host buffers: the host pipeline
    # copies every input in and every output (BF16 y, codes, scales) out, overlapping
    # both PCIe directions with the kernels over three streams
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e = None
    if W.get("adapters") is None:
        from fp4_fake_quant_b200.host import HostPipeline
        pipe = HostPipeline(W["fmt"], W["xs_h"], W["groups"], W["n_groups"], device=dev)
        pipe.run()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a, b = E(), E()
        a.record(stream)
        for _ in range(e2e_steps):
            pipe.run()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([a.elapsed_time(b) / e2e_steps], dev)[0]
        e2e = {"value": weak_scaling_value(step_bytes, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": pipe.h2d_bytes, "d2h_bytes_per_step": pipe.d2h_bytes,
               "steps": e2e_steps, "ms_per_step": e2e_ms,
               "how": "fp4_fake_quant_b200.host.HostPipeline: pinned host in/out, row chunks "
                      "over 3 streams, H2D / kernel / D2H overlapped"}
        del pipe

    pack = pack_timing(W, 20, 3, flush_buf if flush_buf is not None else (lambda: None))
    peak, peak_kind = peaks()
    achieved = W["fq_bytes"] / (kern_ms * 1e-3) / 1e9
    clocks = clk.summary()
    if W["fmt"] == "q4k_mse":
        tops, how = fp32_peak_tops(dev, clocks.get("sm_max_mhz"))
        ach = numel * MSE_OPS_PER_ELEM / (kern_ms * 1e-3) / 1e12
        roofline = {"bound": "alu", "achieved": ach, "peak": tops, "unit": "TOP/s",
                    "frac": ach / tops, "traffic": traffic_for(W["kernel"], W["name"]),
                    "peak_source": f"derived: {how}",
                    "ops_per_element": MSE_OPS_PER_ELEM, "kernel": W["kernel"],
                    "ops_per_launch": numel * MSE_OPS_PER_ELEM, "launch_us": kern_ms * 1e3,
                    "hbm": {"achieved": achieved, "peak": peak, "unit": "GB/s",
                            "frac": achieved / peak}}
    else:
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": traffic_for(W["kernel"], W["name"]),
                    "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                    "kernel": W["kernel"], "bytes_per_launch": W["fq_bytes"],
                    "launch_us": kern_ms * 1e3}
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded stand-ins for real weights and activations)",
        "config": {"workload": W["desc"], "format": W["fmt"], "tensors": W["n_tensors"],
                   "elements_per_step": numel, "bytes_per_step": step_bytes,
                   "input": "fp32" if W["in_bytes"] == 4 else "bf16",
                   "l2": (f"L2 flushed before every step ({in_bytes / 1e6:.0f} MB of input "
                          f"< 2x the {l2 / 1e6:.0f} MB L2): write a 2xL2 buffer, then read "
                          f"another, so L2 holds only clean lines") if flush_buf is not None else
                         (f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB of input vs "
                          f"{l2 / 1e6:.0f} MB); no flush between steps"),
                   "parallelism": f"replicas x{world} (weak scaling, no collective)"},
        "gelem_per_s": world * numel / (ms_per_step * 1e-3) / 1e9,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps * W["launches"],
        "clocks": clocks,
    }
    if pack is not None:
        result["pack_only"] = pack
    del W, flush_buf
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_per_format:
        result["per_format"] = per_format(qf, dev, args, l2, clocks.get("sm_max_mhz"))
        result["export"] = export_timing(qf, dev)
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_rows_frac)
    if "per_format" in result:
        # last key of the line, so that a reader that keeps only its tail sees every workload
        result["per_format_summary"] = format_summary(args.workload, result, peak)
    return result


def _rows_part(frac: float) -> str:
    """Words for a row sample: all rows, or the leading fraction of them."""
    return "all rows" if frac >= 1 else f"the first {frac:.3g} of the rows"


def _r(v, nd=3):
    """Round to `nd` significant digits (None stays None)."""
    if v is None:
        return None
    return float(f"{v:.{nd}g}")


def format_summary(headline: str, result: dict, peak: float) -> dict:
    """Compact per-workload figures: [fused_us, fused_frac, step_us, step_frac], where
    fused is the fake-quant+pack launch alone and step the workload's whole step through
    its one-call entry point (NVFP4: amax + fused pass; LoRA: merge + amax + fused
    pass); fractions are of the measured HBM copy peak, at the algorithmic bytes."""
    out = {"cols": ["fused_us", "fused_frac", "step_us", "step_frac"], "peak_GB/s": peak}
    r = result["roofline"]
    step_frac = result["value"] / result["n_gpus"] / peak
    out[headline] = [_r(r["launch_us"]), _r(r["hbm"]["frac"] if r["bound"] == "alu" else r["frac"]),
                     _r(result["ms_per_step"] * 1e3), _r(step_frac)]
    moe, ste = {}, None
    for name, d in result["per_format"].items():
        if "one_call_step_us" in d:
            su, sg = d["one_call_step_us"], d["one_call_step_GB/s"]
        elif "step_us" in d:
            su, sg = d["step_us"], d["step_GB/s"]
        else:
            su, sg = d["fused_us"], d["fused_GB/s"]
        out[name] = [_r(d["fused_us"]), _r(d["fused_frac_of_hbm_peak"]), _r(su), _r(sg / peak)]
        if "alu_bound" in d:
            out[name + "_alu_frac"] = _r(d["alu_bound"]["frac"])
        if "one_expert_at_a_time_us" in d:
            moe[d["format"]] = [_r(d["fused_us"]), _r(d["one_expert_at_a_time_graph_us"]),
                                _r(d["one_expert_at_a_time_us"])]
        if "ste_identity_us" in d:
            ste = [_r(d["ste_identity_us"]), _r(d["ste_identity_GB/s"] / peak),
                   _r(d["ste_clipped_us"]), _r(d["ste_clipped_GB/s"] / peak)]
    packs = {name: _r(d["pack_only"]["frac_of_hbm_peak"]) for name, d in result["per_format"].items()
             if "pack_only" in d}
    if "pack_only" in result:
        packs = {headline: _r(result["pack_only"]["frac_of_hbm_peak"]), **packs}
    if packs:
        out["pack_only_frac"] = packs
    if moe:
        out["moe_grouped_vs_per_expert_us"] = {"cols": ["grouped", "per_expert_graph",
                                                        "per_expert_eager"], **moe}
    if ste is not None:
        out["ste_tied"] = {"cols": ["identity_us", "identity_frac", "clipped_us",
                                    "clipped_frac"], "v": ste}
    return out


def graph_timed(fn, iters, flush):
    """Median device time (ms) of `fn` captured once in a CUDA graph and replayed, so
    the host's launch rate is not what is measured; None if capture fails."""
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()                                    # fills the host-side caches
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        t = timed_calls(g.replay, iters, 2, flush)
        del g
        return t
    except Exception:                               # noqa: BLE001 (reported as unavailable)
        torch.cuda.synchronize()
        return None


class L2Flush:
    """Evicts the timed kernel's data from L2 between timed calls.

    It writes a buffer of twice the L2 size, then reads a second one of that size.
    The read writes back the dirty lines the write left, so L2 holds only clean
    lines when the timed region starts.  Otherwise the timed kernel would pay for
    writing back up to a whole L2 of the flush's own data.  That costs a kernel of
    tens of MB nearly as much as its own traffic."""

    def __init__(self, dev, l2: int):
        self.w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(2 * l2 // 8, dtype=torch.int64, device=dev)

    def __call__(self):
        self.w.add_(1)
        self.r.max()


def pack_timing(W, iters, warm, flush):
    """The pack-only launch (codes and scales, no BF16 dequant) of a workload that has
    one, timed like the fused pass; its algorithmic bytes are the input read plus
    PACK_BYTES per element.  Run after a whole step, so an NVFP4 amax is real."""
    if "pack" not in W:
        return None
    t = timed_calls(W["pack"], iters, warm, flush)
    gbs = W["numel"] * (W["in_bytes"] + PACK_BYTES[W["fmt"]]) / (t * 1e-3) / 1e9
    return {"us": t * 1e3, "GB/s": gbs, "frac_of_hbm_peak": gbs / peaks()[0],
            "bytes_per_element": W["in_bytes"] + PACK_BYTES[W["fmt"]]}


def timed_calls(fn, iters, warm, flush):
    """Median device time (ms) of `fn` over `iters` calls, each after an L2 flush."""
    for _ in range(warm):
        fn()
    times = []
    for _ in range(iters):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return float(statistics.median(times))


def per_format(qf, dev, args, l2, sm_max_mhz=None):
    peak, _ = peaks()
    flush = L2Flush(dev, l2)
    out = {}
    for name in WORKLOADS:
        if name == args.workload:
            continue
        W = make_workload(name, qf, dev)
        it, warm = args.pf_iters, args.pf_warmup
        # the fused pass alone (for the one-launch NVFP4 step: its qf_fakequant part).
        # One whole step runs first, so an NVFP4 tie-group amax holds its real value: with
        # the zeros it starts from, the tensor scale is 0 and every block takes the
        # zero-scale shortcut, which would time less than the pass's real work.
        pre_fn, fq_fn, fq_bytes = W["parts"] if "parts" in W else (W["pre"], W["fq"], W["fq_bytes"])
        run_step(W)
        t_fq = timed_calls(fq_fn, it, warm, flush)
        pack = pack_timing(W, it, warm, flush)
        t_hot = timed_calls(fq_fn, it, warm, lambda: None)
        gbs = fq_bytes / (t_fq * 1e-3) / 1e9
        d = {"format": W["fmt"], "input": "fp32" if W["in_bytes"] == 4 else "bf16",
             "tensors": W["n_tensors"], "elements": W["numel"],
             "fused_us": t_fq * 1e3, "fused_GB/s": gbs, "fused_Gelem/s": W["numel"] / t_fq / 1e6,
             "fused_frac_of_hbm_peak": gbs / peak,
             # back-to-back calls without a flush: a tensor that fits in L2 is read from it
             "fused_hot_l2_us": t_hot * 1e3,
             "fused_hot_l2_GB/s": fq_bytes / (t_hot * 1e-3) / 1e9}
        if pack is not None:
            d["pack_only"] = pack
        if W["fmt"] == "q4k_mse":
            tops, how = fp32_peak_tops(dev, sm_max_mhz)
            ach = W["numel"] * MSE_OPS_PER_ELEM / (t_fq * 1e-3) / 1e12
            d["alu_bound"] = {"ops_per_element": MSE_OPS_PER_ELEM, "achieved_TOP/s": ach,
                              "peak_TOP/s": tops, "frac": ach / tops, "peak_source": how}
        if pre_fn is not None:
            t_pre = timed_calls(pre_fn, it, warm, flush)
            t_step = timed_calls(lambda: run_step(W), it, warm, flush)
            d.update({"amax_us": t_pre * 1e3,
                      "amax_GB/s": W["in_bytes"] * W["numel"] / t_pre / 1e6,
                      "step_us": t_step * 1e3,
                      "step_GB/s": W["step_bytes"] / t_step / 1e6})
        if "one_call" in W:
            t1 = timed_calls(W["one_call"], it, warm, flush)
            d.update({"one_call_step_us": t1 * 1e3,
                      "one_call_step_GB/s": W["step_bytes"] / t1 / 1e6,
                      "one_call_is": "qf_amax_fakequant without a workspace: amax grid, then "
                                     "the fused grid as its programmatic dependent"})
        if "two_call" in W:
            t2 = timed_calls(W["two_call"], it, warm, flush)
            d.update({"step_is": ("qf_amax_fakequant_lora: merge once into y, then NVFP4 in place"
                                  if name == "lora_nvfp4" else
                                  "qf_amax_fakequant, one cooperative launch"),
                      "two_launch_step_us": t2 * 1e3,
                      "two_launch_step_GB/s": W["step_bytes"] / t2 / 1e6})
        if name == "nvfp4_tied":
            # STE backward of the same tensors (reported beside the step, not in it: the
            # identity is an alias in a training step): identity copy, 4 B per element, and
            # the clipped mask, 6 B per element (reads x and grad_y, writes grad_x)
            g = torch.Generator(device=dev).manual_seed(7)
            gys = [(torch.randn(x.shape, generator=g, device=dev) * 1e-3).to(torch.bfloat16)
                   for x in W["xs"]]
            gxs = [torch.empty_like(t) for t in gys]
            am = torch.empty(W["n_groups"], device=dev)
            qf.qf_amax_tied(W["xs"], W["groups"], am)

            def ste(mode):
                for x, gy, gx, grp in zip(W["xs"], gys, gxs, W["groups"]):
                    qf.qf_ste_backward(gy, gx, mode, "nvfp4", x, grp, am)
            t_id = timed_calls(lambda: ste(0), it, warm, flush)
            t_cl = timed_calls(lambda: ste(1), it, warm, flush)
            d.update({"ste_identity_us": t_id * 1e3,
                      "ste_identity_GB/s": 4 * W["numel"] / t_id / 1e6,
                      "ste_clipped_us": t_cl * 1e3,
                      "ste_clipped_GB/s": 6 * W["numel"] / t_cl / 1e6})
            del gys, gxs
        if name.startswith("moe_"):
            xs, fmt = W["xs"], W["fmt"]
            n = len(xs)
            Y, C = W["outs"][:n], W["outs"][n:2 * n]
            S = W["outs"][2 * n:] if fmt != "q4k" else [None] * n
            groups = [2 * (i // 3) + (i % 3 == 2) for i in range(n)]
            amax = torch.ones(2 * (n // 3), device=dev)

            calls = []
            for e in range(n // 3):
                sl = slice(3 * e, 3 * e + 3)
                if fmt == "nvfp4":
                    calls.append(qf.prepare_fakequant(fmt, xs[sl], Y[sl], C[sl], S[sl],
                                                      groups[sl], amax))
                else:
                    calls.append(qf.prepare_fakequant(fmt, xs[sl], Y[sl], C[sl], S[sl]))

            def looped():
                for c in calls:
                    c()
            t_loop = timed_calls(looped, max(3, it // 4), 1, flush)
            t_loop_g = graph_timed(looped, max(3, it // 4), flush)
            d.update({"one_expert_at_a_time_us": t_loop * 1e3, "grouped_speedup": t_loop / t_fq,
                      "one_expert_at_a_time_graph_us": None if t_loop_g is None else t_loop_g * 1e3})
            if fmt == "nvfp4":
                # the whole NVFP4 step one expert at a time (amax of its two tie groups, then
                # its fused pass): two calls per expert, or one qf_amax_fakequant per expert
                # (a 9.4 MB expert takes the single-launch path)
                ws = qf.alloc_workspace(2, dev)
                two, one = [], []
                for e in range(n // 3):
                    sl = slice(3 * e, 3 * e + 3)
                    am_e = torch.empty(2, device=dev)
                    two.append((qf.prepare_amax_tied(xs[sl], [0, 0, 1], am_e),
                                qf.prepare_fakequant(fmt, xs[sl], Y[sl], C[sl], S[sl], [0, 0, 1],
                                                     am_e)))
                    one.append(qf.prepare_amax_fakequant(xs[sl], Y[sl], C[sl], S[sl], [0, 0, 1],
                                                         am_e, workspace=ws))

                def two_loop():
                    for a, b in two:
                        a()
                        b()

                def one_loop():
                    for c in one:
                        c()
                # replayed from CUDA graphs: host launch cost out of the measurement
                t2 = graph_timed(two_loop, max(3, it // 4), flush)
                t1 = graph_timed(one_loop, max(3, it // 4), flush)
                d.update({"step_one_expert_at_a_time_two_calls_graph_us":
                          None if t2 is None else t2 * 1e3,
                          "step_one_expert_at_a_time_one_launch_graph_us":
                          None if t1 is None else t1 * 1e3})
        out[name] = d
        del W
        torch.cuda.empty_cache()
    return out


def export_timing(qf, dev):
    """The engine containers of two workloads, written from the device bytes: pack on the
    GPU, copy to the host, write the file (host-side; the disk is the box's)."""
    import tempfile

    import gguf  # noqa: F401  (imported outside the timed region: the first import takes ~1 s)
    import safetensors.torch  # noqa: F401
    from fp4_fake_quant_b200 import export
    out = {}
    with tempfile.TemporaryDirectory() as d:
        wl = workloads.q4k_weights()
        xs = [x.to(dev) for x in wl["tensors"]]
        cs = [qf.alloc_outputs("q4k", x, want_y=False)[1] for x in xs]
        qf.qf_pack("q4k", xs, cs)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        export.save_gguf_q4k(os.path.join(d, "q4k.gguf"),
                             [(f"blk.0.{n}.weight", c, x.shape[0], x.shape[1])
                              for n, c, x in zip(("ffn_down", "ffn_up"), cs, xs)])
        dt = time.perf_counter() - t0
        nb = sum(c.numel() for c in cs)
        out["gguf_q4k"] = {"bytes": nb, "s": dt, "MB/s": nb / dt / 1e6,
                           "what": "Q4_K down + up blocks: D2H copy + GGUF write"}
        del xs, cs
        wl = workloads.nvfp4_tied(with_grads=False)
        xs = [x.to(dev) for x in wl["tensors"]]
        ng = wl["n_groups"]
        amax = torch.empty(ng, device=dev)
        outs = [qf.alloc_outputs("nvfp4", x, want_y=False) for x in xs]
        qf.qf_amax_tied(xs, wl["groups"], amax)
        qf.qf_pack("nvfp4", xs, [o[1] for o in outs], [o[2] for o in outs], wl["groups"], amax)
        torch.cuda.synchronize()
        am = amax.cpu().numpy()
        t0 = time.perf_counter()
        tensors = {}
        for n, x, o, g in zip(wl["names"], xs, outs, wl["groups"]):
            tensors.update(export.compressed_tensors_nvfp4(f"layers.0.{n}", o[1], o[2],
                                                           x.shape[0], x.shape[1], float(am[g])))
        export.save_safetensors(os.path.join(d, "nvfp4.safetensors"), tensors)
        dt = time.perf_counter() - t0
        nb = sum(v.numel() * v.element_size() for v in tensors.values())
        out["safetensors_nvfp4"] = {"bytes": nb, "s": dt, "MB/s": nb / dt / 1e6,
                                    "what": "NVFP4 tied projections, compressed-tensors tensors: "
                                            "D2H copy + safetensors write"}
        del xs, outs
    torch.cuda.empty_cache()
    return out


def _host_cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return max(1, os.cpu_count() or 1)


def _oracle_pass(fmt, tensors, threads):
    """The oracle, as it stands, over `tensors` (CPU BF16), their rows split into
    `threads` contiguous ranges run on as many host threads (the oracle's C calls
    release the GIL; rows are independent and the NVFP4 amax is a max of maxes, so
    the bytes are those of one call).  Returns the elements processed."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    n = 0
    with ThreadPoolExecutor(max_workers=threads) as pool:
        for x in tensors:
            rows = x.shape[0]
            cuts = [rows * i // threads for i in range(threads + 1)]
            parts = [x[a:b] for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
            if fmt == "nvfp4":
                am = max(pool.map(oracle.amax, parts))
                list(pool.map(lambda p: oracle.nvfp4(p, am), parts))
            elif fmt == "mxfp4":
                list(pool.map(oracle.mxfp4, parts))
            else:
                list(pool.map(lambda p: oracle.q4k(p, mse=fmt == "q4k_mse"), parts))
            n += x.numel()
    return n


def cpu_baseline(name, frac):
    """The oracle, as it stands, on the first `frac` of the rows of each tensor: on every
    host core of this process's affinity mask, and on one core."""
    import oracle
    oracle.build()
    gen = {"w4a4": workloads.mxfp4_w4a4, "q4k": workloads.q4k_weights,
           "q4k_mse": workloads.q4k_weights,
           "q4k_f32": lambda: workloads.q4k_weights(dtype="f32"),
           "nvfp4_tied": lambda: workloads.nvfp4_tied(with_grads=False),
           "nvfp4_tied_f32": lambda: workloads.nvfp4_tied(with_grads=False, dtype="f32"),
           "nvfp4_weight": workloads.nvfp4_weight, "activation": workloads.nvfp4_activation,
           "moe_nvfp4": workloads.moe_experts, "moe_mxfp4": workloads.moe_experts,
           "moe_q4k": workloads.moe_experts}
    fmt = {"w4a4": "mxfp4", "q4k": "q4k", "q4k_mse": "q4k_mse", "q4k_f32": "q4k",
           "moe_mxfp4": "mxfp4", "moe_q4k": "q4k"}.get(name, "nvfp4")
    if name not in gen:                     # LoRA: the oracle's fake-quant of the bases alone
        gen[name] = lambda: workloads.nvfp4_tied(with_grads=False)
    wl = gen[name]()
    sample = [x[: max(1, int(x.shape[0] * frac))] for x in wl["tensors"]]
    cores = _host_cores()
    t0 = time.perf_counter()
    n = _oracle_pass(fmt, sample, cores)
    dt_all = time.perf_counter() - t0
    one = [x[: max(1, x.shape[0] // 4)] for x in sample]         # a quarter of it on one core
    t0 = time.perf_counter()
    n1 = _oracle_pass(fmt, one, 1)
    dt_one = time.perf_counter() - t0
    bpe = BYTES_PER_ELEM[fmt] + sample[0].element_size() - 2      # FP32 input reads 4 B
    return {"value": n * bpe / dt_all / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{_rows_part(frac)} of every tensor ({n} elements), scalar C, "
                      f"rows split over {cores} host threads, {dt_all:.1f} s",
            "single_core_value": n1 * bpe / dt_one / 1e9,
            "single_core_sample": f"a quarter of that sample ({n1} elements) on one thread, "
                                  f"{dt_one:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world):
    """The oracle as the reference arm: the same metric on the host cores, each step a
    bounded sample of the workload sized so warmup + steps take about a minute."""
    import oracle
    oracle.build()
    wl = workloads.mxfp4_w4a4()
    n_total = sum(t.numel() for t in wl["tensors"])
    cores = _host_cores()
    per_step_s = 60.0 / max(1, args.steps + args.warmup)
    # ~80 ns per element per core for the scalar oracle
    frac = min(1.0, max(1.0 / 4096, per_step_s / (n_total * 80e-9 / cores)))
    sample = [t[: max(1, int(t.shape[0] * frac))] for t in wl["tensors"]]
    n = sum(t.numel() for t in sample)

    def step():
        _oracle_pass("mxfp4", sample, cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = n * BYTES_PER_ELEM["mxfp4"] / dt / 1e9
    desc = (f"oracle (scalar C) on {_rows_part(frac)} of W and A ({n} elements) "
            f"per step, rows split over {cores} host threads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "MXFP4 W4A4: weight BF16 12288x4096 + activations BF16 "
                                   "32768x4096 (bounded row sample per step)",
                       "format": "mxfp4", "parallelism": "host cores, rank 0 only"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="w4a4", choices=WORKLOADS)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--pf-iters", type=int, default=100)
    ap.add_argument("--pf-warmup", type=int, default=20)
    ap.add_argument("--cpu-rows-frac", type=float, default=0.5)
    ap.add_argument("--no-per-format", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
