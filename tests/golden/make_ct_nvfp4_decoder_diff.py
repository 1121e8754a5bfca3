"""Writes ct_nvfp4_decoder_diff.json: the number of elements on which compressed-tensors'
own NVFP4 decompressor differs from the oracle's dequantized BF16 y, for the NVFP4 tied
projections (Q 4096x4096, K and V 1024x4096 sharing one tensor scale; gate and up
14336x4096 sharing another; N(0, 0.02) with 0.1% of entries x20), at full size and at
1/64 of the rows.

Only the oracle (codes, block scales, y), the seeded input generators and
compressed-tensors (the engine library's decoder) are called.  The exported tensors
follow compressed-tensors' NVFP4 layout: weight_packed (codes), weight_scale (E4M3
bytes) and weight_global_scale = 2688 / amax in FP32.

    python tests/golden/make_ct_nvfp4_decoder_diff.py
"""
import json
import os
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads  # noqa: E402


def decoder_diff(x, amax_g, pool):
    """(elements, differing elements, max difference in BF16 units of the oracle's y)."""
    from compressed_tensors.compressors.nvfp4.base import NVFP4PackedCompressor
    from compressed_tensors.quantization import QuantizationScheme
    from compressed_tensors.quantization.quant_scheme import PRESET_SCHEMES

    rows, cols = x.shape
    cuts = [rows * i // 16 for i in range(17)]
    parts = list(pool.map(lambda ab: oracle.nvfp4(x[ab[0]:ab[1]], amax_g)[:3],
                          [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]))
    y = np.concatenate([p[0] for p in parts])
    codes = np.concatenate([p[1] for p in parts])
    scales = np.concatenate([p[2] for p in parts])
    g = np.float32(2688.0) / np.float32(amax_g)
    sd = {"weight_packed": torch.from_numpy(codes).view(rows, cols // 2),
          "weight_scale": torch.from_numpy(scales).view(torch.float8_e4m3fn).view(rows, cols // 16),
          "weight_global_scale": torch.tensor([g], dtype=torch.float32)}
    scheme = QuantizationScheme(targets=["Linear"], **PRESET_SCHEMES["NVFP4"])
    w = NVFP4PackedCompressor.decompress(sd, scheme)["weight"].to(torch.bfloat16)
    wb = w.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    diff = wb != y
    ours = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).float().numpy()
    theirs = w.float().numpy().reshape(-1)
    ulp = np.maximum(np.abs(ours), np.float32(2.0 ** -126)) * np.float32(2.0 ** -7)
    return int(y.size), int(diff.sum()), float(np.max(np.abs(theirs - ours) / ulp))


def measure(rows_scale, pool):
    wl = workloads.nvfp4_tied(rows_scale=rows_scale, with_grads=False)
    am = oracle.tied_amax(wl["tensors"], wl["groups"], wl["n_groups"])
    n = d = 0
    worst = 0.0
    for x, gi in zip(wl["tensors"], wl["groups"]):
        a, b, c = decoder_diff(x, float(am[gi]), pool)
        n, d, worst = n + a, d + b, max(worst, c)
    return {"elements": n, "differing": d, "max_bf16_units": worst}


def main():
    with ThreadPoolExecutor(max_workers=max(1, len(os.sched_getaffinity(0)))) as pool:
        out = {"workload": "NVFP4 tied Q/K/V + gate/up, N(0, 0.02) with 0.1% x20 outliers, seed 3",
               "decoder": "compressed_tensors NVFP4PackedCompressor.decompress",
               "rows_scale_1": measure(1.0, pool),
               "rows_scale_1_64": measure(1 / 64, pool)}
    with open(os.path.join(HERE, "ct_nvfp4_decoder_diff.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out))


if __name__ == "__main__":
    main()
