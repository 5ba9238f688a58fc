"""QLoRA linear layer (NF4 + double quantization + LoRA) for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``lib/libqlora.so`` (CUDA, built from
``csrc/`` by ``build.py``); ``qlora`` is its thin ctypes binding and ``inputs``
draws seeded synthetic workloads.
"""
from .qlora import (CODEBOOK_NF4, CODEBOOK_UNIFORM4, NF4Weight, PagedBuffer, QLoraError,  # noqa: F401
                    codebook_tables, fp8_thresholds, lib, nf4_code_buckets,
                    nf4_table, nf4_thresholds, qlora_dequant, qlora_device_error,
                    qlora_linear_bwd, qlora_merge_lora,
                    qlora_linear_bwd_workspace_size, qlora_linear_fwd,
                    qlora_linear_fwd_workspace_size, qlora_profile_events, qlora_quantize_nf4_dq,
                    qlora_quantize_workspace_size, qlora_adamw_state_bytes, qlora_adamw_step)
