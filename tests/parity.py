"""Comparison rules between the CUDA path and the fp64 oracle, and helpers
that run one workload instance through both.

Tolerances:
  * 16-bit y: per element |g - o| <= 4e-3 |o|.  Only where o is zero or
    below the format's smallest normal number (fp16 subnormals, where the
    fixed spacing makes rounding alone exceed 4e-3 relative) may g instead be
    within one unit in the last place of RNE(o).  For normal outputs RNE
    itself is within half a unit, 2^-8 < 4e-3 relative in bf16 and 2^-11 in
    fp16, so the relative bound is the whole test there;
  * residual_out: within one ulp of RNE(r), r the exact fp64 sum;
  * FP8 codes: within one e4m3 step (adjacent codes in value order);
  * FP8 scales: within 1e-6 relative of amax/448 in fp64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from tensor_allreduce_residual_ar_b200 import workloads as wl

Y_RTOL = 4e-3
SCALE_RTOL = 1e-6
# smallest positive normal number of each 16-bit format
MIN_NORMAL = {"bf16": 2.0 ** -126, "fp16": 2.0 ** -14}


def ordinal16(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ordinal8(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.int32)
    return np.where(c & 0x80, -(c & 0x7F), c)


def check_y(gpu_bits: np.ndarray, y64: np.ndarray, dtype: str, what: str = "y"):
    """Per-element check of 16-bit outputs against the fp64 oracle.  Returns
    the largest and the 99.99th-percentile relative error over non-zero
    oracle values, the number of elements that needed the one-ulp clause
    (all of them zero or subnormal in the output format), and how many
    elements lay in that range at all."""
    dt = wl.DTYPE_CODE[dtype]
    g = oracle.decode16(gpu_bits, dt)
    rel_ok = np.abs(g - y64) <= Y_RTOL * np.abs(y64)
    tiny = np.abs(y64) < MIN_NORMAL[dtype]
    ulp_ok = tiny & (np.abs(ordinal16(gpu_bits) - ordinal16(oracle.round16(y64, dt))) <= 1)
    bad = ~(rel_ok | ulp_ok)
    nbad = int(bad.sum())
    if nbad:
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {nbad} elements outside tolerance; first {idx.tolist()}: "
                             f"gpu {g[bad][:5]} oracle {y64[bad][:5]}")
    nz = y64 != 0
    rel = np.abs(g[nz] - y64[nz]) / np.abs(y64[nz])
    normal = ~tiny
    rel_n = np.abs(g[normal] - y64[normal]) / np.abs(y64[normal])
    return {"max_rel": float(rel.max()) if rel.size else 0.0,
            "max_rel_normal": float(rel_n.max()) if rel_n.size else 0.0,
            "p9999_rel": float(np.quantile(rel, 0.9999)) if rel.size else 0.0,
            "ulp_clause": int((~rel_ok & ulp_ok).sum()),
            "tiny": int(tiny.sum())}


def check_res(gpu_bits: np.ndarray, r64: np.ndarray, dtype: str):
    dt = wl.DTYPE_CODE[dtype]
    d = np.abs(ordinal16(gpu_bits) - ordinal16(oracle.round16(r64, dt)))
    if int(d.max(initial=0)) > 1:
        idx = np.argwhere(d > 1)[:5]
        raise AssertionError(f"residual_out: {int((d > 1).sum())} elements beyond 1 ulp; first {idx.tolist()}")
    return {"exact": float((d == 0).mean()) if d.size else 1.0}


def check_fp8(q_gpu: np.ndarray, s_gpu: np.ndarray, y64: np.ndarray, group: int = 128):
    q_o, s64, _ = oracle.quant_fp8_group(y64, group)
    d = np.abs(ordinal8(q_gpu) - ordinal8(q_o))
    if int(d.max(initial=0)) > 1:
        idx = np.argwhere(d > 1)[:5]
        raise AssertionError(f"fp8: {int((d > 1).sum())} codes beyond one e4m3 step; first {idx.tolist()}")
    s_gpu = s_gpu.astype(np.float64)
    zero = s64 == 0
    if not np.all(s_gpu[zero] == 0):
        raise AssertionError("fp8: non-zero scale for an all-zero group")
    rel = np.abs(s_gpu[~zero] - s64[~zero]) / s64[~zero]
    if rel.size and rel.max() > SCALE_RTOL:
        raise AssertionError(f"fp8 scales: max rel err {rel.max():.3e} > {SCALE_RTOL}")
    return {"codes_exact": float((d == 0).mean()) if d.size else 1.0,
            "scale_max_rel": float(rel.max()) if rel.size else 0.0}


def to_bits(t: torch.Tensor) -> np.ndarray:
    return wl.bits(t.cpu())


# ----------------------------------------------------------------------------
# oracle side
# ----------------------------------------------------------------------------

def oracle_norm(inp: wl.NormInputs, rows=None):
    """Oracle y and r, optionally for a subset of rows only."""
    parts = [wl.bits(p) for p in inp.partials]
    res = wl.bits(inp.residual) if inp.residual is not None else None
    if rows is not None:
        parts = [p[rows] for p in parts]
        res = res[rows] if res is not None else None
    return oracle.ar_add_rmsnorm(parts, res, wl.bits(inp.weight), inp.eps, inp.gemma,
                                 wl.DTYPE_CODE[inp.dtype])


def oracle_qk(inp: wl.QKInputs, rows=None):
    shards = [wl.bits(x) for x in inp.qkv]
    if rows is not None:
        shards = [s[rows] for s in shards]
    return oracle.qk_norm_sharded(shards, wl.bits(inp.q_weight), wl.bits(inp.k_weight),
                                  inp.q_size, inp.kv_size, inp.eps, wl.DTYPE_CODE[inp.dtype])
