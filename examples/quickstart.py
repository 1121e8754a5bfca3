"""Quick start: NVFP4 fake-quant + pack of a Q/K/V projection group that shares one
tensor scale, then a compressed-tensors checkpoint shard written from the packed bytes.

Run from any directory with a B200 visible; it writes model-00001.safetensors there."""
import torch

import fp4_fake_quant_b200 as qf
from fp4_fake_quant_b200 import export

q, k, v = (torch.randn(r, 4096, device="cuda", dtype=torch.bfloat16) * 0.02
           for r in (4096, 1024, 1024))
xs, groups = [q, k, v], [0, 0, 0]                  # Q, K, V share one NVFP4 tensor scale
outs = [qf.alloc_outputs("nvfp4", x) for x in xs]  # (y BF16, packed codes, E4M3 scales)
amax = torch.empty(1, device="cuda")
ws = qf.alloc_workspace(1)
qf.qf_amax_fakequant(xs, [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs],
                     groups, amax, workspace=ws)
qf.qf_workspace_check(ws)                          # raises if the grid barrier gave up
# forward: use outs[i][0] (the dequantized weight); backward: the gradient passes straight through
tensors = {}
for name, x, (y, c, s) in zip(("q_proj", "k_proj", "v_proj"), xs, outs):
    tensors.update(export.compressed_tensors_nvfp4(f"layers.0.self_attn.{name}", c, s,
                                                   x.shape[0], x.shape[1], amax.item()))
export.save_safetensors("model-00001.safetensors", tensors)
