"""PyTorch custom operators over the library's calls.

    torch.ops.ar_b200.add_rmsnorm(partials, residual, weight, eps, gemma) -> (y, residual_out)
    torch.ops.ar_b200.add_rmsnorm_out_only(partials, residual, weight, eps, gemma) -> y
    torch.ops.ar_b200.add_rmsnorm_fp8_group(partials, residual, weight, eps, gemma)
        -> (q, scales, y, residual_out)
    torch.ops.ar_b200.qk_norm_sharded(qkv, q_weight, k_weight, q_size, kv_size, eps)
        -> (q_out, k_out)

The tensor-parallel form, one partial per rank and a communicator
registered with ``comm.register`` (its id is the last argument):

    torch.ops.ar_b200.tp_add_rmsnorm(partial, residual, weight, eps, gemma, comm) -> (y, residual_out)
    torch.ops.ar_b200.tp_add_rmsnorm_out_only(partial, residual, weight, eps, gemma, comm) -> y
    torch.ops.ar_b200.tp_add_rmsnorm_fp8_group(partial, residual, weight, eps, gemma, comm)
        -> (q, scales, y, residual_out)
    torch.ops.ar_b200.tp_qk_norm_sharded(qkv, q_weight, k_weight, q_size, kv_size, eps, comm)
        -> (q_out, k_out)        # this rank's shard; only per-token sums of squares cross ranks

They are collective: every rank calls them in the same order.

They let torch programs use the fused step as one operator: outputs are
allocated on the inputs' device by torch's caching allocator and computed by
the library's kernels on the current stream, so the calls can be captured in
CUDA graphs; the fake implementations give shapes and dtypes for tracing and
check the arguments the library would reject.  `residual` may be None (the
no-residual form); `add_rmsnorm_out_only` is the output-only (dead-residual)
form.  Inference only: there is no autograd formula.  CUDA tensors only.
"""
from __future__ import annotations

import torch

from . import binding as ar

_DT = (torch.bfloat16, torch.float16)


def _check_norm(partials, residual, weight):
    if len(partials) < 1 or len(partials) > 16:
        raise ValueError("1 to 16 partials are supported")
    x = partials[0]
    H = weight.shape[-1]
    if weight.dim() != 1 or x.shape[-1] != H or H % 8 != 0:
        raise ValueError("weight must be [H] with H a multiple of 8 and partials [..., H]")
    for t in list(partials) + ([residual] if residual is not None else []):
        if t.shape != x.shape or t.dtype != x.dtype or t.device != x.device:
            raise ValueError("partials and residual must share shape, dtype and device")
    if x.dtype not in _DT or weight.dtype != x.dtype:
        raise TypeError("bf16 or fp16 tensors of one dtype are supported")
    return x, H


@torch.library.custom_op("ar_b200::add_rmsnorm", mutates_args=(), device_types="cuda")
def add_rmsnorm(partials: list[torch.Tensor], residual: torch.Tensor | None, weight: torch.Tensor,
                eps: float, gemma: bool) -> tuple[torch.Tensor, torch.Tensor]:
    x, _ = _check_norm(partials, residual, weight)
    y, r = torch.empty_like(x), torch.empty_like(x)
    ar.ar_add_rmsnorm(list(partials), residual, weight, y, r, eps=eps, gemma=gemma)
    return y, r


@add_rmsnorm.register_fake
def _add_rmsnorm_fake(partials, residual, weight, eps, gemma):
    x, _ = _check_norm(partials, residual, weight)
    return torch.empty_like(x), torch.empty_like(x)


@torch.library.custom_op("ar_b200::add_rmsnorm_out_only", mutates_args=(), device_types="cuda")
def add_rmsnorm_out_only(partials: list[torch.Tensor], residual: torch.Tensor | None,
                         weight: torch.Tensor, eps: float, gemma: bool) -> torch.Tensor:
    x, _ = _check_norm(partials, residual, weight)
    y = torch.empty_like(x)
    ar.ar_add_rmsnorm(list(partials), residual, weight, y, None, eps=eps, gemma=gemma)
    return y


@add_rmsnorm_out_only.register_fake
def _add_rmsnorm_out_only_fake(partials, residual, weight, eps, gemma):
    x, _ = _check_norm(partials, residual, weight)
    return torch.empty_like(x)


@torch.library.custom_op("ar_b200::add_rmsnorm_fp8_group", mutates_args=(), device_types="cuda")
def add_rmsnorm_fp8_group(partials: list[torch.Tensor], residual: torch.Tensor | None,
                          weight: torch.Tensor, eps: float,
                          gemma: bool) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    x, H = _check_norm(partials, residual, weight)
    if H % 128 != 0:
        raise ValueError("H must be a multiple of the group size 128")
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty((*x.shape[:-1], H // 128), dtype=torch.float32, device=x.device)
    y, r = torch.empty_like(x), torch.empty_like(x)
    ar.ar_add_rmsnorm_quant_fp8_group(list(partials), residual, weight, q, s, y, r, eps=eps, gemma=gemma)
    return q, s, y, r


@add_rmsnorm_fp8_group.register_fake
def _add_rmsnorm_fp8_group_fake(partials, residual, weight, eps, gemma):
    x, H = _check_norm(partials, residual, weight)
    if H % 128 != 0:
        raise ValueError("H must be a multiple of the group size 128")
    return (torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device),
            torch.empty((*x.shape[:-1], H // 128), dtype=torch.float32, device=x.device),
            torch.empty_like(x), torch.empty_like(x))


def _check_qk(qkv, q_weight, k_weight, q_size, kv_size):
    W = len(qkv)
    if W < 1 or W > 16 or q_size % W or kv_size % W:
        raise ValueError("1 to 16 shards dividing q_size and kv_size")
    qs, ks = q_size // W, kv_size // W
    if qs % 8 or ks % 8:
        raise ValueError("per-shard q and k widths must be multiples of 8")
    x = qkv[0]
    for t in qkv:
        if t.shape != x.shape or t.dtype != x.dtype or t.shape[-1] != qs + 2 * ks:
            raise ValueError("every shard must be [..., q_size/W + 2*kv_size/W] of one dtype")
    if tuple(q_weight.shape) != (q_size,) or tuple(k_weight.shape) != (kv_size,):
        raise ValueError("q_weight must be [q_size] and k_weight [kv_size]")
    if x.dtype not in _DT or q_weight.dtype != x.dtype or k_weight.dtype != x.dtype:
        raise TypeError("bf16 or fp16 tensors of one dtype are supported")
    return x, qs, ks


@torch.library.custom_op("ar_b200::qk_norm_sharded", mutates_args=(), device_types="cuda")
def qk_norm_sharded(qkv: list[torch.Tensor], q_weight: torch.Tensor, k_weight: torch.Tensor,
                    q_size: int, kv_size: int,
                    eps: float) -> tuple[list[torch.Tensor], list[torch.Tensor]]:
    x, qs, ks = _check_qk(qkv, q_weight, k_weight, q_size, kv_size)
    lead = x.shape[:-1]
    qo = [torch.empty((*lead, qs), dtype=x.dtype, device=x.device) for _ in qkv]
    ko = [torch.empty((*lead, ks), dtype=x.dtype, device=x.device) for _ in qkv]
    ar.qk_norm_sharded(list(qkv), q_weight, k_weight, qo, ko, q_size, kv_size, eps=eps)
    return qo, ko


@qk_norm_sharded.register_fake
def _qk_norm_sharded_fake(qkv, q_weight, k_weight, q_size, kv_size, eps):
    x, qs, ks = _check_qk(qkv, q_weight, k_weight, q_size, kv_size)
    lead = x.shape[:-1]
    return ([x.new_empty((*lead, qs)) for _ in qkv], [x.new_empty((*lead, ks)) for _ in qkv])


# ---------------------------------------------------------------------------
# tensor-parallel form: this rank's partial, all-reduced over the ranks of a
# registered communicator inside the fused call
# ---------------------------------------------------------------------------

def _comm(comm: int):
    from . import comm as C
    return C.lookup(comm)


@torch.library.custom_op("ar_b200::tp_add_rmsnorm", mutates_args=(), device_types="cuda")
def tp_add_rmsnorm(partial: torch.Tensor, residual: torch.Tensor | None, weight: torch.Tensor,
                   eps: float, gemma: bool, comm: int) -> tuple[torch.Tensor, torch.Tensor]:
    x, _ = _check_norm([partial], residual, weight)
    y, r = torch.empty_like(x), torch.empty_like(x)
    _comm(comm).allreduce_add_rmsnorm(partial, residual, weight, y, r, eps=eps, gemma=gemma)
    return y, r


@tp_add_rmsnorm.register_fake
def _tp_add_rmsnorm_fake(partial, residual, weight, eps, gemma, comm):
    x, _ = _check_norm([partial], residual, weight)
    return torch.empty_like(x), torch.empty_like(x)


@torch.library.custom_op("ar_b200::tp_add_rmsnorm_out_only", mutates_args=(), device_types="cuda")
def tp_add_rmsnorm_out_only(partial: torch.Tensor, residual: torch.Tensor | None, weight: torch.Tensor,
                            eps: float, gemma: bool, comm: int) -> torch.Tensor:
    x, _ = _check_norm([partial], residual, weight)
    y = torch.empty_like(x)
    _comm(comm).allreduce_add_rmsnorm(partial, residual, weight, y, None, eps=eps, gemma=gemma)
    return y


@tp_add_rmsnorm_out_only.register_fake
def _tp_add_rmsnorm_out_only_fake(partial, residual, weight, eps, gemma, comm):
    x, _ = _check_norm([partial], residual, weight)
    return torch.empty_like(x)


@torch.library.custom_op("ar_b200::tp_add_rmsnorm_fp8_group", mutates_args=(), device_types="cuda")
def tp_add_rmsnorm_fp8_group(partial: torch.Tensor, residual: torch.Tensor | None, weight: torch.Tensor,
                             eps: float, gemma: bool,
                             comm: int) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    x, H = _check_norm([partial], residual, weight)
    if H % 128 != 0:
        raise ValueError("H must be a multiple of the group size 128")
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty((*x.shape[:-1], H // 128), dtype=torch.float32, device=x.device)
    y, r = torch.empty_like(x), torch.empty_like(x)
    _comm(comm).allreduce_add_rmsnorm_quant_fp8_group(partial, residual, weight, q, s, out_y=y,
                                                      residual_out=r, eps=eps, gemma=gemma)
    return q, s, y, r


@tp_add_rmsnorm_fp8_group.register_fake
def _tp_add_rmsnorm_fp8_group_fake(partial, residual, weight, eps, gemma, comm):
    x, H = _check_norm([partial], residual, weight)
    if H % 128 != 0:
        raise ValueError("H must be a multiple of the group size 128")
    return (torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device),
            torch.empty((*x.shape[:-1], H // 128), dtype=torch.float32, device=x.device),
            torch.empty_like(x), torch.empty_like(x))


def _check_tp_qk(qkv, q_weight, k_weight, q_size, kv_size, world):
    if q_size % world or kv_size % world:
        raise ValueError(f"q_size and kv_size must be multiples of the world size {world}")
    qs, ks = q_size // world, kv_size // world
    if qs % 8 or ks % 8:
        raise ValueError("per-rank q and k widths must be multiples of 8")
    if qkv.shape[-1] != qs + 2 * ks:
        raise ValueError("this rank's qkv must be [..., q_size/W + 2*kv_size/W]")
    if tuple(q_weight.shape) != (q_size,) or tuple(k_weight.shape) != (kv_size,):
        raise ValueError("q_weight must be [q_size] and k_weight [kv_size]")
    if qkv.dtype not in _DT or q_weight.dtype != qkv.dtype or k_weight.dtype != qkv.dtype:
        raise TypeError("bf16 or fp16 tensors of one dtype are supported")
    return qs, ks


@torch.library.custom_op("ar_b200::tp_qk_norm_sharded", mutates_args=(), device_types="cuda")
def tp_qk_norm_sharded(qkv: torch.Tensor, q_weight: torch.Tensor, k_weight: torch.Tensor, q_size: int,
                       kv_size: int, eps: float, comm: int) -> tuple[torch.Tensor, torch.Tensor]:
    c = _comm(comm)
    qs, ks = _check_tp_qk(qkv, q_weight, k_weight, q_size, kv_size, c.world)
    lead = qkv.shape[:-1]
    qo = torch.empty((*lead, qs), dtype=qkv.dtype, device=qkv.device)
    ko = torch.empty((*lead, ks), dtype=qkv.dtype, device=qkv.device)
    c.qk_norm_sharded(qkv, q_weight, k_weight, qo, ko, q_size, kv_size, eps=eps)
    return qo, ko


@tp_qk_norm_sharded.register_fake
def _tp_qk_norm_sharded_fake(qkv, q_weight, k_weight, q_size, kv_size, eps, comm):
    # the world size is the communicator's; the shard's width fixes it
    row = qkv.shape[-1]
    world = (q_size + 2 * kv_size) // row if row else 0
    if world < 1 or world * row != q_size + 2 * kv_size:
        raise ValueError("qkv's width must be (q_size + 2*kv_size) / W for the communicator's W")
    qs, ks = _check_tp_qk(qkv, q_weight, k_weight, q_size, kv_size, world)
    lead = qkv.shape[:-1]
    return qkv.new_empty((*lead, qs)), qkv.new_empty((*lead, ks))
