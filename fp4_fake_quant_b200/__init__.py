"""B200-native deployment-aligned simulated quantization (NVFP4 / MXFP4 / Q4_K).

The product is libqf.so (C ABI in include/qf.h, CUDA kernels for sm_100a in
csrc/); ``binding`` is its thin ctypes binding with the same entry-point names.
"""
from .binding import (QF_MXFP4, QF_NVFP4, QF_Q4K, QF_X_BF16, QF_X_F32, FORMATS, EXPORTS, QfError,
                      alloc_outputs, alloc_workspace, output_sizes, prepare_amax_fakequant,
                      prepare_amax_fakequant_lora, prepare_amax_tied, prepare_amax_tied_lora, prepare_fakequant,
                      prepare_fakequant_lora, Prepared, qf_amax_fakequant,
                      qf_amax_fakequant_lora, qf_amax_fakequant_noalloc, qf_amax_tied, qf_amax_tied_lora, qf_fakequant,
                      qf_fakequant_lora, qf_lora_merge, qf_pack, qf_ste_backward,
                      qf_noalloc_check, qf_test_barrier_timeout, qf_workspace_check,
                      workspace_bytes, lib)

__all__ = ["QF_NVFP4", "QF_MXFP4", "QF_Q4K", "QF_X_BF16", "QF_X_F32", "FORMATS", "EXPORTS",
           "QfError", "alloc_outputs", "alloc_workspace", "output_sizes",
           "prepare_amax_fakequant", "prepare_amax_fakequant_lora", "prepare_amax_tied", "prepare_amax_tied_lora",
           "prepare_fakequant", "prepare_fakequant_lora", "Prepared", "qf_amax_fakequant",
           "qf_amax_fakequant_lora", "qf_amax_fakequant_noalloc", "qf_amax_tied", "qf_amax_tied_lora", "qf_fakequant",
           "qf_fakequant_lora", "qf_lora_merge", "qf_pack", "qf_ste_backward",
           "qf_noalloc_check", "qf_test_barrier_timeout", "qf_workspace_check",
           "workspace_bytes", "lib"]
