"""Seeded synthetic inputs for the five workloads.

This module draws random numbers and casts them to 16-bit formats; it holds
none of the method's arithmetic, and both the CUDA path and the CPU oracle
consume what it produces.  Everything is generated on the CPU with
``torch.Generator`` so any test can regenerate the exact bits.

Recipe (shapes and distributions of the five workloads; N(mu, s) means mean
mu and standard deviation s):

* tiny      T=16, H=4096, W=2 bf16 partials N(0,1), residual N(0,1),
            weight N(1,0.1), eps=1e-6, standard RMSNorm, y and residual_out.
* decode    T in {1,2,4,8,16,32,64,80}, H=8192, W=4 partials N(0,0.5) in
            bf16 and fp16, residual N(0,1), weight N(0,0.1), Gemma (1+w),
            eps=1e-6, y and residual_out.
* prefill   T=8192, H=4096, W=8 bf16 partials N(0,1/8), residual N(0,1),
            weight N(1,0.1), eps=1e-5, output-only (residual_out not written).
* fp8       T = 1, 2, 4, ..., 32768, H=5120, W=4 bf16 partials N(0,1),
            residual N(0,1), weight N(1,0.1), eps=1e-6, group 128 e4m3 with
            y and residual_out also emitted in bf16.
* qk        T in {1,64,2048}, W=8 shards of [q_size/W | kv_size/W |
            kv_size/W] with q_size=6144, kv_size=1024, bf16 N(0,1), weights
            N(1,0.1), eps=1e-6.

Values are drawn in fp32 and cast with round-to-nearest-even.  The seed of a
workload instance is 20260000 + 1000 * workload_index + T; draws happen in
the order partials 0..W-1, residual, weight (qk: shards 0..W-1, q_weight,
k_weight).  ``eps`` is handed to the library as an fp32 value, so the float
actually used is ``float32(eps)``; the oracle receives that same value.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

WORKLOAD_INDEX = {"tiny": 0, "decode": 1, "prefill": 2, "fp8": 3, "qk": 4}

_TORCH_DTYPE = {"bf16": torch.bfloat16, "fp16": torch.float16}
DTYPE_CODE = {"bf16": 0, "fp16": 1}


@dataclass(frozen=True)
class NormWorkload:
    name: str
    Ts: tuple
    H: int
    W: int
    dtypes: tuple
    partial: tuple          # (mean, std)
    residual: tuple | None  # (mean, std) or None for the no-residual form
    weight: tuple
    gemma: bool
    eps: float
    write_residual: bool
    fp8: bool = False
    group: int = 128


@dataclass(frozen=True)
class QKWorkload:
    name: str
    Ts: tuple
    W: int
    q_size: int
    kv_size: int
    dtypes: tuple
    act: tuple
    weight: tuple
    eps: float


TINY = NormWorkload("tiny", (16,), 4096, 2, ("bf16",), (0.0, 1.0), (0.0, 1.0),
                    (1.0, 0.1), False, 1e-6, True)
DECODE = NormWorkload("decode", (1, 2, 4, 8, 16, 32, 64, 80), 8192, 4, ("bf16", "fp16"),
                      (0.0, 0.5), (0.0, 1.0), (0.0, 0.1), True, 1e-6, True)
PREFILL = NormWorkload("prefill", (8192,), 4096, 8, ("bf16",), (0.0, 0.125), (0.0, 1.0),
                       (1.0, 0.1), False, 1e-5, False)
FP8 = NormWorkload("fp8", tuple(2 ** k for k in range(16)), 5120, 4, ("bf16",),
                   (0.0, 1.0), (0.0, 1.0), (1.0, 0.1), False, 1e-6, True, fp8=True)
QK = QKWorkload("qk", (1, 64, 2048), 8, 6144, 1024, ("bf16",), (0.0, 1.0), (1.0, 0.1), 1e-6)

WORKLOADS = {w.name: w for w in (TINY, DECODE, PREFILL, FP8, QK)}


def seed_for(name: str, T: int) -> int:
    return 20260000 + 1000 * WORKLOAD_INDEX[name] + int(T)


def eps32(eps: float) -> float:
    """The eps value the library actually receives (an fp32 parameter)."""
    return float(np.float32(eps))


def _draw(gen: torch.Generator, shape, mean: float, std: float, dtype: str) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x.to(_TORCH_DTYPE[dtype])


def bits(t: torch.Tensor) -> np.ndarray:
    """16-bit tensor -> numpy uint16 bit patterns (no copy of values)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class NormInputs:
    partials: list
    residual: torch.Tensor | None
    weight: torch.Tensor
    T: int
    H: int
    W: int
    dtype: str
    eps: float
    gemma: bool
    write_residual: bool
    extra: dict = field(default_factory=dict)


def make_norm_inputs(wl: NormWorkload, T: int, dtype: str | None = None, *, seed: int | None = None,
                     W: int | None = None, H: int | None = None,
                     residual: bool | None = None, device: str = "cpu") -> NormInputs:
    """Inputs of one instance of a norm workload.  ``W``, ``H``, ``residual``
    and ``seed`` may be overridden for edge-case tests (same distributions).
    ``device="cuda"`` draws the same distributions with the device generator
    (other values than the CPU draw; used only for timing)."""
    dtype = dtype or wl.dtypes[0]
    W = wl.W if W is None else W
    H = wl.H if H is None else H
    has_res = (wl.residual is not None) if residual is None else residual
    gen = torch.Generator(device=device).manual_seed(seed_for(wl.name, T) if seed is None else seed)
    parts = [_draw(gen, (T, H), *wl.partial, dtype) for _ in range(W)]
    res = _draw(gen, (T, H), *(wl.residual or (0.0, 1.0)), dtype) if has_res else None
    wt = _draw(gen, (H,), *wl.weight, dtype)
    return NormInputs(parts, res, wt, T, H, W, dtype, eps32(wl.eps), wl.gemma,
                      wl.write_residual)


@dataclass
class QKInputs:
    qkv: list
    q_weight: torch.Tensor
    k_weight: torch.Tensor
    T: int
    W: int
    q_size: int
    kv_size: int
    dtype: str
    eps: float


def make_qk_inputs(wl: QKWorkload, T: int, dtype: str | None = None, *, seed: int | None = None,
                   W: int | None = None, q_size: int | None = None,
                   kv_size: int | None = None, device: str = "cpu") -> QKInputs:
    dtype = dtype or wl.dtypes[0]
    W = wl.W if W is None else W
    q_size = wl.q_size if q_size is None else q_size
    kv_size = wl.kv_size if kv_size is None else kv_size
    gen = torch.Generator(device=device).manual_seed(seed_for(wl.name, T) if seed is None else seed)
    row = q_size // W + 2 * (kv_size // W)
    shards = [_draw(gen, (T, row), *wl.act, dtype) for _ in range(W)]
    qw = _draw(gen, (q_size,), *wl.weight, dtype)
    kw = _draw(gen, (kv_size,), *wl.weight, dtype)
    return QKInputs(shards, qw, kw, T, W, q_size, kv_size, dtype, eps32(wl.eps))


def norm_bytes(T: int, H: int, W: int, has_res: bool, write_res: bool, elt: int = 2,
               fp8: bool = False, write_y16: bool = True, group: int = 128) -> int:
    """Algorithmic HBM bytes of one call: each input read once, each output
    written once, the weight counted once."""
    reads = (W + (1 if has_res else 0)) * T * H * elt + H * elt
    if fp8:
        writes = T * H + T * (H // group) * 4
        writes += T * H * elt if write_y16 else 0
    else:
        writes = T * H * elt
    writes += T * H * elt if write_res else 0
    return reads + writes


def qk_bytes(T: int, W: int, q_size: int, kv_size: int, elt: int = 2) -> int:
    """q and k of every shard read once and written once; both weight
    vectors read once; v untouched."""
    return 2 * T * (q_size + kv_size) * elt + (q_size + kv_size) * elt
