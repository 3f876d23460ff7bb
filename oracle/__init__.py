"""fp64 CPU oracle for the fused W-way reduce + residual add + RMSNorm step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never loads it, and it never loads the CUDA library: the two
share no code.  Inputs come from the seeded generators in
``tensor_allreduce_residual_ar_b200.workloads``, which hold none of the
method's arithmetic.

The arithmetic lives in ``oracle.c`` (plain C, fp64, built with gcc; see the
header of that file for the passages each function follows).  This module
builds it on first use and wraps it with ctypes over numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py``; nothing in
this oracle is "parity unpinned" except the two facts the pages leave
undefined (the metric behind their 2.7e-3 parity figure, and AITER's own FP8
scale layout), which no test can compare against.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
FP16 = 1


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared library with gcc (no -ffast-math, no
    FMA contraction, no -march: IEEE fp64 on any x86-64 host)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _configure(lib):
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.oracle_decode16.restype = ctypes.c_double
    lib.oracle_decode16.argtypes = [ctypes.c_uint16, ctypes.c_int]
    lib.oracle_round16.restype = ctypes.c_uint16
    lib.oracle_round16.argtypes = [ctypes.c_double, ctypes.c_int]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_ar_add_rmsnorm.restype = None
    lib.oracle_ar_add_rmsnorm.argtypes = [P, ctypes.c_int, P, P, i64, i64,
                                          ctypes.c_double, ctypes.c_int,
                                          ctypes.c_int, P, P, P]
    lib.oracle_quant_fp8_group.restype = None
    lib.oracle_quant_fp8_group.argtypes = [P, i64, i64, ctypes.c_int, P, P, P]
    lib.oracle_qk_norm_sharded.restype = None
    lib.oracle_qk_norm_sharded.argtypes = [P, ctypes.c_int, P, P, i64, i64, i64,
                                           ctypes.c_double, ctypes.c_int, P, P]
    for name in ("oracle_round16_array", "oracle_decode16_array"):
        fn = getattr(lib, name)
        fn.restype = None
        fn.argtypes = [P, i64, ctypes.c_int, P]
    for name in ("oracle_e4m3_encode_array", "oracle_e4m3_decode_array"):
        fn = getattr(lib, name)
        fn.restype = None
        fn.argtypes = [P, i64, P]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
        return _lib


def compile_variant(source_text: str, out_path: str) -> str:
    """Compile an edited copy of oracle.c (used by the mutation test, which
    plants slips in copies of the source to show the pins catch them)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    "-fno-fast-math", "-w", "-o", out_path, src, "-lm"], check=True)
    return out_path


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every call of this module to another build."""
    global _lib
    saved = _load()
    with _lock:
        _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bit patterns, got {a.dtype}")
    return a


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _ptr_array(arrs):
    return (ctypes.c_void_p * len(arrs))(*[_ptr(a) for a in arrs])


# ----------------------------------------------------------------------------
# scalar / array format helpers
# ----------------------------------------------------------------------------

def decode16(bits, dtype: int) -> np.ndarray:
    """16-bit patterns -> exact fp64 values."""
    bits = _u16(bits)
    out = np.empty(bits.shape, np.float64)
    _load().oracle_decode16_array(_ptr(bits), bits.size, dtype, _ptr(out))
    return out


def round16(x, dtype: int) -> np.ndarray:
    """fp64 values -> 16-bit patterns, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_round16_array(_ptr(x), x.size, dtype, _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """fp64 values -> e4m3fn codes, round to nearest even, saturating."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float64)
    _load().oracle_e4m3_decode_array(_ptr(codes), codes.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# the method
# ----------------------------------------------------------------------------

def ar_add_rmsnorm(partials, residual, weight, eps: float, gemma: bool, dtype: int,
                   want_r: bool = True, want_inv: bool = False):
    """W partials [T, H] (uint16 bits), residual [T, H] or None, weight [H].

    Returns dict with ``y`` (fp64 [T, H], unrounded), ``r`` (exact fp64 sum,
    if want_r) and ``inv`` (fp64 [T] = 1/sqrt(ms+eps), if want_inv).
    """
    parts = [_u16(p) for p in partials]
    W = len(parts)
    T, H = parts[0].shape
    for p in parts:
        assert p.shape == (T, H)
    res = _u16(residual) if residual is not None else None
    if res is not None:
        assert res.shape == (T, H)
    wt = _u16(weight)
    assert wt.shape == (H,)
    y = np.empty((T, H), np.float64)
    r = np.empty((T, H), np.float64) if want_r else None
    inv = np.empty((T,), np.float64) if want_inv else None
    _load().oracle_ar_add_rmsnorm(
        _ptr_array(parts), W, _ptr(res) if res is not None else None, _ptr(wt),
        T, H, float(eps), int(bool(gemma)), int(dtype), _ptr(y),
        _ptr(r) if r is not None else None, _ptr(inv) if inv is not None else None)
    out = {"y": y}
    if r is not None:
        out["r"] = r
    if inv is not None:
        out["inv"] = inv
    return out


def quant_fp8_group(y, group: int = 128):
    """y fp64 [T, H] -> (q uint8 [T, H], scales64 [T, H/group], scales32)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    T, H = y.shape
    assert H % group == 0
    q = np.empty((T, H), np.uint8)
    s64 = np.empty((T, H // group), np.float64)
    s32 = np.empty((T, H // group), np.float32)
    _load().oracle_quant_fp8_group(_ptr(y), T, H, int(group), _ptr(q), _ptr(s64), _ptr(s32))
    return q, s64, s32


def qk_norm_sharded(qkv, q_weight, k_weight, q_size: int, kv_size: int, eps: float,
                    dtype: int):
    """W shard buffers [T, q_size/W + 2*kv_size/W] -> (q_out [W,T,qs], k_out [W,T,ks])."""
    shards = [_u16(x) for x in qkv]
    W = len(shards)
    T = shards[0].shape[0]
    qs, ks = q_size // W, kv_size // W
    for x in shards:
        assert x.shape == (T, qs + 2 * ks)
    qw, kw = _u16(q_weight), _u16(k_weight)
    assert qw.shape == (q_size,) and kw.shape == (kv_size,)
    q_out = np.empty((W, T, qs), np.float64)
    k_out = np.empty((W, T, ks), np.float64)
    _load().oracle_qk_norm_sharded(_ptr_array(shards), W, _ptr(qw), _ptr(kw), T,
                                   int(q_size), int(kv_size), float(eps), int(dtype),
                                   _ptr(q_out), _ptr(k_out))
    return q_out, k_out
