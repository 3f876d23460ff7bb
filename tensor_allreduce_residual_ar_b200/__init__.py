"""Fused W-way reduce + residual add + RMSNorm for NVIDIA B200 (sm_100a).

The compute lives in a C-ABI CUDA library (``csrc/``, header
``include/ar_rmsnorm.h``); this package is its thin Python binding, plus the
same calls as PyTorch custom operators (``torch.ops.ar_b200.*``, see
``torch_ops``).
"""
from .binding import (  # noqa: F401
    AR_BF16, AR_FP16, ARError, ar_add_rmsnorm, ar_add_rmsnorm_quant_fp8_group,
    ar_device_status, ar_plan_force, ar_plan_load, ar_plan_query, ar_plan_table_size,
    ar_status_string, ar_test_withhold_row,
    library_path, load_library, qk_norm_sharded,
)
from . import torch_ops  # noqa: F401,E402  (registers torch.ops.ar_b200.*)
