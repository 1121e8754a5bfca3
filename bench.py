#!/usr/bin/env python3
"""Benchmark of the fused fake-quant + pack pass on B200.

Headline workload: MXFP4 W4A4 -- weight BF16 12288x4096 N(0, 0.02) and
activations 8 x 4096 tokens by 4096 hidden, Student-t(3) with 1% of channels
x50 -- quantized in ONE grouped qf_fakequant launch that writes dequantized
BF16, packed E2M1 nibbles and E8M0 block scales.  A step is that launch.

  value      GB/s of algorithmic bytes (read BF16 + write BF16 + codes + scales,
             4.53125 B/element) over the device-timed steps, max over ranks,
             summed over ranks (weak scaling: every rank quantizes its own batch).
  e2e        the same metric through the public API with pinned host buffers:
             host->device copy of the inputs, the call, device->host copy of
             every output, per step.
  roofline   that kernel's achieved GB/s against the measured HBM copy peak.
  cpu_baseline  the oracle (scalar C, one thread) on a bounded sample of the rows.
  per_format NVFP4 (tied QKV/gate-up, amax + fake-quant), Q4_K (down/up), NVFP4
             4096^2 weight (L2 flushed), MoE grouped vs looped, timed per call.

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
                  "q4k": 2 + 2 + 144 / 256}
WORKLOAD = ("MXFP4 W4A4: weight BF16 12288x4096 N(0,0.02) + activations BF16 32768x4096 "
            "(8x4096 tokens) Student-t(3), 1% channels x50; one grouped fake-quant+pack launch")
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    def __init__(self, index: int):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _names(self, mask):
        nv = self.nv
        table = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
                 "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
                 "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
                 "display_clock_setting": 0x100}
        return {k for k, v in table.items() if mask & v}

    def _run(self):
        while not self._stop.is_set():
            self.sample_once()
            time.sleep(0.002)

    def sample_once(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self._names(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def __enter__(self):
        self.sample_once()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self.t.join()
        self.sample_once()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def csrc_digest() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "fp4_fake_quant_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this exact source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(kernel)
        if e and e.get("csrc_sha") == csrc_digest() and e.get("workload") == workload:
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import fp4_fake_quant_b200 as qf
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    wl = workloads.mxfp4_w4a4(seed=1 + 1000 * rank)
    xs_h = [t.pin_memory() for t in wl["tensors"]]
    xs = [t.to(dev, non_blocking=True) for t in xs_h]
    outs = [qf.alloc_outputs("mxfp4", x) for x in xs]
    ys, cs, ss = [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs]
    numel = sum(x.numel() for x in xs)
    step_bytes = numel * BYTES_PER_ELEM["mxfp4"]
    torch.cuda.synchronize()

    def step():
        qf.qf_fakequant("mxfp4", xs, ys, cs, ss)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    per_launch_ms = [a.elapsed_time(b) for a, b in ev]
    kern_ms = float(np.mean(per_launch_ms))
    t = torch.tensor([total_ms, kern_ms], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    total_ms, kern_ms = float(t[0]), float(t[1])
    ms_per_step = total_ms / args.steps
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API with pinned host buffers
    ys_h = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in ys]
    cs_h = [torch.empty(c.shape, dtype=c.dtype, pin_memory=True) for c in cs]
    ss_h = [torch.empty(s.shape, dtype=s.dtype, pin_memory=True) for s in ss]
    e2e_steps = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        for xd, xh in zip(xs, xs_h):
            xd.copy_(xh, non_blocking=True)
        qf.qf_fakequant("mxfp4", xs, ys, cs, ss)
        for d, h in zip(ys + cs + ss, ys_h + cs_h + ss_h):
            h.copy_(d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([a.elapsed_time(b) / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(e2e_ms, op=torch.distributed.ReduceOp.MAX)
    h2d = sum(x.numel() * x.element_size() for x in xs)
    d2h = sum(t.numel() * t.element_size() for t in ys + cs + ss)
    e2e = {"value": world * step_bytes / (float(e2e_ms) * 1e-3) / 1e9, "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "ms_per_step": float(e2e_ms)}

    peak, peak_kind = peaks()
    achieved = step_bytes / (kern_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"{peak_kind} HBM copy bandwidth",
                "kernel": "k_fp4<MXFP4> (qf_fakequant, grouped over W and A)",
                "bytes_per_launch": step_bytes,
                "traffic": traffic_for("k_fp4_mxfp4", "w4a4")}

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; Student-t / normal stand-ins for real weights and activations)",
        "config": {"workload": WORKLOAD, "format": "mxfp4", "elements_per_step": numel,
                   "bytes_per_element": BYTES_PER_ELEM["mxfp4"],
                   "l2": f"inputs larger than L2 ({2 * numel / 1e6:.0f} MB of BF16 vs "
                         f"{L2_BYTES / 1e6:.0f} MB); no flush between steps",
                   "parallelism": f"replicas x{world}"},
        "gelem_per_s": world * numel / (ms_per_step * 1e-3) / 1e9,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_per_format:
        result["per_format"] = per_format(qf, dev, args)
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(wl, args.cpu_rows_frac)
    return result


def timed_calls(fn, iters, warm, flush=None):
    """Median device time of `fn` over `iters` calls, each on a cold L2 when `flush`."""
    for _ in range(warm):
        fn()
    times = []
    for _ in range(iters):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return float(statistics.median(times))


def per_format(qf, dev, args):
    peak, _ = peaks()
    scratch = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        scratch.add_(1)

    out = {}
    it, warm = args.pf_iters, 3

    def entry(fmt, numel, ms, extra=None):
        gbs = numel * BYTES_PER_ELEM[fmt] / (ms * 1e-3) / 1e9
        d = {"format": fmt, "elements": numel, "us": ms * 1e3, "GB/s": gbs,
             "Gelem/s": numel / (ms * 1e-3) / 1e9, "frac_of_hbm_peak": gbs / peak}
        if extra:
            d.update(extra)
        return d

    # NVFP4 tied QKV + gate/up: tied amax, then the fused pass (+ STE identity)
    wl = workloads.nvfp4_tied(with_grads=False)
    xs = [t.to(dev) for t in wl["tensors"]]
    del wl
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    amax = torch.empty(2, device=dev)
    so = torch.empty(2, device=dev)
    n = sum(x.numel() for x in xs)
    f_amax = lambda: qf.qf_amax_tied(xs, [0, 0, 0, 1, 1], amax)
    f_fq = lambda: qf.qf_fakequant("nvfp4", xs, [o[0] for o in outs], [o[1] for o in outs],
                                   [o[2] for o in outs], [0, 0, 0, 1, 1], amax, so)
    t_amax = timed_calls(f_amax, it, warm, flush)
    t_fq = timed_calls(f_fq, it, warm, flush)
    t_both = timed_calls(lambda: (f_amax(), f_fq()), it, warm, flush)
    g = torch.empty_like(xs[3])
    t_ste = timed_calls(lambda: qf.qf_ste_backward(xs[3], g, mode=0), it, warm, flush)
    out["nvfp4_tied_qkv_gateup"] = entry("nvfp4", n, t_fq, {
        "amax_us": t_amax * 1e3, "amax_GB/s": 2 * n / (t_amax * 1e-3) / 1e9,
        "amax_plus_fakequant_us": t_both * 1e3,
        "ste_identity_GB/s": 4 * xs[3].numel() / (t_ste * 1e-3) / 1e9})
    del xs, outs, g

    # Q4_K down + up
    wl = workloads.q4k_weights()
    xs = [t.to(dev) for t in wl["tensors"]]
    del wl
    outs = [qf.alloc_outputs("q4k", x) for x in xs]
    n = sum(x.numel() for x in xs)
    t_q = timed_calls(lambda: qf.qf_fakequant("q4k", xs, [o[0] for o in outs],
                                              [o[1] for o in outs]), it, warm, flush)
    out["q4k_down_up"] = entry("q4k", n, t_q)
    del xs, outs

    # NVFP4 4096x4096 weight (fits in L2: flushed before every call)
    wl = workloads.nvfp4_weight()
    x = wl["tensors"][0].to(dev)
    y, c, s = qf.alloc_outputs("nvfp4", x)
    am1 = torch.empty(1, device=dev)
    qf.qf_amax_tied([x], [0], am1)
    t1 = timed_calls(lambda: qf.qf_fakequant("nvfp4", [x], [y], [c], [s], [0], am1), it, warm,
                     flush)
    t1b = timed_calls(lambda: (qf.qf_amax_tied([x], [0], am1),
                               qf.qf_fakequant("nvfp4", [x], [y], [c], [s], [0], am1)),
                      it, warm, flush)
    out["nvfp4_weight_4096"] = entry("nvfp4", x.numel(), t1, {"amax_plus_fakequant_us": t1b * 1e3})
    del x, y, c, s

    # MoE: 128 experts x {gate, up, down}, grouped vs one expert at a time
    wl = workloads.moe_experts()
    xs = [t.to(dev) for t in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    del wl
    n = sum(x.numel() for x in xs)
    am = torch.empty(ng, device=dev)
    for fmt in ("nvfp4", "mxfp4", "q4k"):
        outs = [qf.alloc_outputs(fmt, x) for x in xs]
        Y, C, S = [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs]
        if fmt == "nvfp4":
            qf.qf_amax_tied(xs, groups, am)
        kw = {"groups": groups, "group_amax": am} if fmt == "nvfp4" else {}
        tg = timed_calls(lambda: qf.qf_fakequant(fmt, xs, Y, C, S, **kw), max(3, it // 4), 2, flush)

        def looped():
            for e in range(128):
                sl = slice(3 * e, 3 * e + 3)
                kw2 = {"groups": groups[sl], "group_amax": am} if fmt == "nvfp4" else {}
                qf.qf_fakequant(fmt, xs[sl], Y[sl], C[sl], S[sl], **kw2)
        tl = timed_calls(looped, max(3, it // 4), 1, flush)
        out[f"moe128_{fmt}"] = entry(fmt, n, tg, {"looped_us": tl * 1e3,
                                                 "grouped_speedup": tl / tg})
        del outs, Y, C, S

    # NVFP4 activation 32768x4096 with tracked amax (amax pass + fused pass)
    wl = workloads.nvfp4_activation()
    a = wl["tensors"][0].to(dev)
    del wl
    y, c, s = qf.alloc_outputs("nvfp4", a)
    cur, tracked = torch.empty(1, device=dev), torch.zeros(1, device=dev)
    ta = timed_calls(lambda: (qf.qf_amax_tied([a], [0], cur, tracked),
                              qf.qf_fakequant("nvfp4", [a], [y], [c], [s], [0], tracked)),
                     it, warm, flush)
    out["nvfp4_activation_tracked"] = entry("nvfp4", a.numel(), ta,
                                            {"includes": "amax pass + fused pass"})
    del a, y, c, s, scratch
    torch.cuda.empty_cache()
    return out


def cpu_baseline(wl, frac):
    """The oracle, as it stands, on the first `frac` of the rows of each tensor."""
    import oracle
    oracle.build()
    n = 0
    t0 = time.perf_counter()
    for x in wl["tensors"]:
        r = max(1, int(x.shape[0] * frac))
        oracle.mxfp4(x[:r])
        n += r * x.shape[1]
    dt = time.perf_counter() - t0
    return {"value": n * BYTES_PER_ELEM["mxfp4"] / dt / 1e9, "unit": UNIT, "cores": 1,
            "kind": "oracle",
            "sample": f"first {frac:.3g} of the rows of W and A ({n} elements), scalar C, "
                      f"one thread, {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    import oracle
    oracle.build()
    wl = workloads.mxfp4_w4a4(rows_scale=1.0)
    n_total = sum(t.numel() for t in wl["tensors"])
    # per-step sample sized so that warmup + steps take about a minute of host time
    per_step_s = 60.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(1.0 / 4096, per_step_s / (n_total * 80e-9)))
    sample = [t[: max(1, int(t.shape[0] * frac))] for t in wl["tensors"]]
    n = sum(t.numel() for t in sample)

    def step():
        for t in sample:
            oracle.mxfp4(t)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = n * BYTES_PER_ELEM["mxfp4"] / dt / 1e9
    desc = (f"oracle (scalar C, one thread) on the first {frac:.3g} of the rows of W and A "
            f"({n} elements) per step")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": WORKLOAD, "format": "mxfp4",
                                            "parallelism": "host, rank 0 only"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
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
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--pf-iters", type=int, default=20)
    ap.add_argument("--cpu-rows-frac", type=float, default=0.5)
    ap.add_argument("--no-per-format", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
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
