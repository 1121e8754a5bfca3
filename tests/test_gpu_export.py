"""From device bytes to engine files: the CUDA path's packed outputs, written by
fp4_fake_quant_b200.export and read back by llama.cpp's gguf reader and by
safetensors, decode to the CUDA path's own fake-quant output (QATFactory project
page, Method, "Export")."""
import numpy as np
import pytest
import torch

import fp4_fake_quant_b200 as qf
import workloads
from fp4_fake_quant_b200 import export
from gpu_helpers import DEV, bits

pytestmark = pytest.mark.gpu
gguf = pytest.importorskip("gguf")


def _bf16_bits(a32):
    return workloads.bf16_bits(torch.from_numpy(np.ascontiguousarray(a32, np.float32))
                               .to(torch.bfloat16)).reshape(-1)


def test_q4k_device_bytes_to_gguf(tmp_path):
    wl = workloads.q4k_weights(rows_scale=1 / 16)
    xs = [x.to(DEV) for x in wl["tensors"]]
    outs = [qf.alloc_outputs("q4k", x) for x in xs]
    qf.qf_fakequant("q4k", xs, [o[0] for o in outs], [o[1] for o in outs])
    torch.cuda.synchronize()
    names = ["blk.0.ffn_down.weight", "blk.0.ffn_up.weight"]
    path = str(tmp_path / "model.gguf")
    export.save_gguf_q4k(path, [(n, o[1], x.shape[0], x.shape[1])
                                for n, o, x in zip(names, outs, xs)])
    got = {t.name: t for t in gguf.GGUFReader(path).tensors}
    for n, o in zip(names, outs):
        deq = gguf.quants.dequantize(np.asarray(got[n].data), got[n].tensor_type)
        assert np.array_equal(_bf16_bits(deq.reshape(-1)), bits(o[0])), n


def test_nvfp4_device_bytes_to_safetensors(tmp_path):
    from compressed_tensors.compressors.nvfp4.helpers import unpack_fp4_from_uint8
    from safetensors.torch import load_file

    wl = workloads.nvfp4_tied(rows_scale=1 / 16, with_grads=False)
    xs = [x.to(DEV) for x in wl["tensors"]]
    groups, ng = wl["groups"], wl["n_groups"]
    amax, so = torch.empty(ng, device=DEV), torch.empty(ng, device=DEV)
    outs = [qf.alloc_outputs("nvfp4", x) for x in xs]
    qf.qf_amax_fakequant(xs, [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs],
                         groups, amax, group_scale_out=so, workspace=qf.alloc_workspace(ng, DEV))
    torch.cuda.synchronize()
    am, st = amax.cpu().numpy(), so.cpu().numpy()
    tensors = {}
    for name, x, o, g in zip(wl["names"], xs, outs, groups):
        tensors.update(export.compressed_tensors_nvfp4(f"layer.{name}", o[1], o[2], x.shape[0],
                                                       x.shape[1], float(am[g])))
    path = str(tmp_path / "model.safetensors")
    export.save_safetensors(path, tensors)
    back = load_file(path)
    for name, x, o, g in zip(wl["names"], xs, outs, groups):
        rows, cols = x.shape
        v = unpack_fp4_from_uint8(back[f"layer.{name}.weight_packed"], rows, cols,
                                  dtype=torch.float32).numpy()
        sb = back[f"layer.{name}.weight_scale"].to(torch.float32).numpy()
        S = (np.repeat(sb, 16, axis=1) * np.float32(st[g])).astype(np.float32)
        assert np.array_equal(_bf16_bits(v * S), bits(o[0])), name
        gs = float(back[f"layer.{name}.weight_global_scale"][0])
        assert gs == float(np.float32(2688.0) / np.float32(am[g]))
    # Q, K and V share one global scale; gate and up share another
    gsc = [float(back[f"layer.{n}.weight_global_scale"][0]) for n in wl["names"]]
    assert gsc[0] == gsc[1] == gsc[2] and gsc[3] == gsc[4]
