"""QLoRA NF4 + double-quant linear layer for one B200 (sm_100a).

Thin Python binding over the C ABI of ``libqlora_nf4.so`` (declared in
``include/qlora_nf4.h``).  Every function here only marshals arguments: torch
tensors supply device memory and the current CUDA stream, and every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if
the library is missing or no sm_100 device is current, calls raise.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    QLORA_OUT_BF16,
    QLORA_OUT_FP32,
    QloraError,
    exported_symbols,
    lib_path,
    load,
    qlora_debug_record,
    qlora_dequant,
    qlora_dropout_apply,
    qlora_launch_count,
    qlora_device_status,
    qlora_linear_bwd,
    qlora_linear_bwd_dropout,
    qlora_linear_fwd,
    qlora_linear_fwd_dropout,
    qlora_linear_fwd_noalloc,
    qlora_merge_adapter,
    qlora_nf4_codebook,
    qlora_quantize_nf4_dq,
    qlora_quantize_nf4_dq_fp8,
    qlora_quantize_nf4,
    qlora_selftest_device_timeout,
    qlora_strerror,
    qlora_timing_collect,
    qlora_timing_enable,
    qlora_workspace_bytes,
    qlora_workspace_bytes_dropout,
)
