"""Engine-native containers around the packed bytes.

The QATFactory project page (Method, "Export") has the trained weights exported in
each engine's own format: vLLM compressed-tensors checkpoints for NVFP4 and MXFP4,
and a llama.cpp GGUF file for Q4_K.  The NVFP4 activation scales tracked during
training go into the checkpoint too, so the server needs no calibration.  The
quantization itself is done on the device by qf_pack / qf_fakequant; this module
only names the bytes and writes the containers on the host.

compressed-tensors tensors of one linear layer ``prefix`` (packed formats):
  NVFP4  ``prefix.weight_packed``  uint8 [rows, cols/2], element 2i in the low nibble
         ``prefix.weight_scale``   float8_e4m3fn [rows, cols/16]: the E4M3 block scales
         ``prefix.weight_global_scale``  float32 [1]
         ``prefix.input_global_scale``   float32 [1], from the tracked activation amax
  MXFP4  ``prefix.weight_packed``  uint8 [rows, cols/2]
         ``prefix.weight_scale``   uint8 [rows, cols/32]: E8M0 bytes (exponent + 127)
compressed-tensors stores the reciprocal of the FP32 tensor scale as a "global
scale" and dequantizes as code * block_scale / global_scale.  The global scale of
a tensor with amax a is 2688 / a in FP32 (2688 = 448 * 6), and 1 when that is not
finite (a == 0: every block scale is then 0).

GGUF: every Q4_K tensor is the sequence of 144-byte blocks qf_pack writes.  The
header, the key/value metadata and the tensor infos are written by the ``gguf``
package (llama.cpp's own writer); it is imported only when a GGUF file is written.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np
import torch

E2M1_MAX_X_E4M3_MAX = 6.0 * 448.0


def nvfp4_global_scale(amax: float) -> float:
    """compressed-tensors global scale of a tie group: FP32 2688 / amax (1 if not finite)."""
    a = np.float32(amax)
    with np.errstate(divide="ignore", over="ignore"):
        g = np.float32(E2M1_MAX_X_E4M3_MAX) / a
    return float(g) if np.isfinite(g) else 1.0


def _host_u8(t: torch.Tensor, shape) -> torch.Tensor:
    if t.dtype != torch.uint8:
        raise TypeError("packed codes and scales are uint8 tensors")
    return t.detach().to("cpu").contiguous().view(shape)


def compressed_tensors_nvfp4(prefix: str, codes: torch.Tensor, scales: torch.Tensor, rows: int,
                             cols: int, weight_amax: float,
                             input_amax: Optional[float] = None) -> Dict[str, torch.Tensor]:
    """The compressed-tensors tensors of one NVFP4 linear layer.

    codes / scales: the outputs of qf_pack / qf_fakequant for a [rows, cols] weight;
    weight_amax: its tie group's amax (the one the scales were derived from);
    input_amax: the tracked activation amax of the layer's input, or None."""
    if cols % 16:
        raise ValueError("NVFP4 needs cols % 16 == 0")
    out = {
        f"{prefix}.weight_packed": _host_u8(codes, (rows, cols // 2)),
        f"{prefix}.weight_scale": _host_u8(scales, (rows, cols // 16)).view(torch.float8_e4m3fn),
        f"{prefix}.weight_global_scale": torch.tensor([nvfp4_global_scale(weight_amax)],
                                                      dtype=torch.float32),
    }
    if input_amax is not None:
        out[f"{prefix}.input_global_scale"] = torch.tensor([nvfp4_global_scale(input_amax)],
                                                           dtype=torch.float32)
    return out


def compressed_tensors_mxfp4(prefix: str, codes: torch.Tensor, scales: torch.Tensor, rows: int,
                             cols: int) -> Dict[str, torch.Tensor]:
    """The compressed-tensors tensors of one MXFP4 linear layer."""
    if cols % 32:
        raise ValueError("MXFP4 needs cols % 32 == 0")
    return {
        f"{prefix}.weight_packed": _host_u8(codes, (rows, cols // 2)),
        f"{prefix}.weight_scale": _host_u8(scales, (rows, cols // 32)),
    }


def quantization_config(fmt: str, ignore: Sequence[str] = ("lm_head",),
                        activations: bool = True) -> dict:
    """The ``quantization_config`` block of config.json for a compressed-tensors
    checkpoint in ``fmt`` ("nvfp4" or "mxfp4"), built from compressed-tensors' own
    preset schemes (W4A4, or weight-only when ``activations`` is False)."""
    from compressed_tensors.quantization import QuantizationConfig, QuantizationScheme
    from compressed_tensors.quantization.quant_scheme import PRESET_SCHEMES

    preset = {"nvfp4": "NVFP4", "mxfp4": "MXFP4"}[fmt] + ("" if activations else "A16")
    scheme = QuantizationScheme(targets=["Linear"], **PRESET_SCHEMES[preset])
    cfg = QuantizationConfig(config_groups={"group_0": scheme},
                             format=f"{fmt}-pack-quantized", ignore=list(ignore),
                             quantization_status="compressed")
    return cfg.model_dump(mode="json", exclude_none=True)


def save_safetensors(path: str, tensors: Dict[str, torch.Tensor]) -> None:
    """Write a safetensors shard (the container compressed-tensors checkpoints use)."""
    from safetensors.torch import save_file

    save_file({k: v.contiguous() for k, v in tensors.items()}, path, metadata={"format": "pt"})


def save_gguf_q4k(path: str, tensors: Iterable[Tuple[str, torch.Tensor, int, int]],
                  arch: str = "llama", kv: Optional[Dict[str, object]] = None) -> None:
    """Write a GGUF file holding Q4_K tensors.

    tensors: (name, blocks, rows, cols) with blocks the uint8 output of qf_pack for a
    [rows, cols] weight (rows * cols / 256 blocks of 144 bytes).  kv: extra string /
    integer / float metadata."""
    import gguf

    w = gguf.GGUFWriter(path, arch)
    for key, val in (kv or {}).items():
        if isinstance(val, str):
            w.add_string(key, val)
        elif isinstance(val, bool):
            w.add_bool(key, val)
        elif isinstance(val, int):
            w.add_uint32(key, val)
        elif isinstance(val, float):
            w.add_float32(key, val)
        else:
            raise TypeError(f"metadata {key}: unsupported type {type(val).__name__}")
    for name, blocks, rows, cols in tensors:
        if cols % 256:
            raise ValueError(f"{name}: Q4_K needs cols % 256 == 0")
        b = _host_u8(blocks, (rows, cols // 256 * 144)).numpy()
        w.add_tensor(name, b, raw_dtype=gguf.GGMLQuantizationType.Q4_K)
    w.write_header_to_file()
    w.write_kv_data_to_file()
    w.write_tensors_to_file()
    w.close()
