"""Fused W-way reduce + residual add + RMSNorm for NVIDIA B200 (sm_100a).

The compute lives in a C-ABI CUDA library (``csrc/``, headers
``include/ar_rmsnorm.h`` and ``include/ar_comm.h``); this package is its thin
Python binding: the single-GPU calls below, the same calls as PyTorch custom
operators (``torch.ops.ar_b200.*``, see ``torch_ops``), the multi-GPU form
(``comm.Comm`` for one process per GPU, ``comm.CommGroup`` for W ranks run on
one GPU), and a torch.fx rewrite that routes unfused all-reduce + add +
RMSNorm subgraphs to the fused operators (``fx_patterns``).
"""
from .binding import (  # noqa: F401
    AR_BF16, AR_FP16, ARError, ar_add_rmsnorm, ar_add_rmsnorm_quant_fp8_group,
    ar_device_status, ar_plan_force, ar_plan_load, ar_plan_query, ar_plan_table_size,
    ar_status_string, ar_test_withhold_row,
    library_path, load_library, qk_norm_sharded,
)
from . import torch_ops  # noqa: F401,E402  (registers torch.ops.ar_b200.*)
from . import comm  # noqa: F401,E402
