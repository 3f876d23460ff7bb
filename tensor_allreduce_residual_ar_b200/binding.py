"""ctypes binding of the C ABI in ``include/ar_rmsnorm.h``.

Argument marshalling only: shapes, dtypes and device pointers are read from
torch tensors and handed to the C entry points of the same names, on torch's
current CUDA stream unless a stream is given.  Every step of the computation
runs in the library's CUDA kernels; there is no Python or CPU fallback, and a
missing library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

AR_BF16 = 0
AR_FP16 = 1
AR_MAX_W = 16
_DTYPES = {torch.bfloat16: AR_BF16, torch.float16: AR_FP16}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_lib", "libar_rmsnorm.so")
_PLAN_TABLE = os.path.join(_HERE, "plan_table.json")
_lock = threading.Lock()
_lib = None


class ARError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {ar_status_string(status)} (status {status})")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the CUDA library (built by ``tensor_allreduce_residual_ar_b200.build``)
    and its shipped plan table.  Raises if the library is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"CUDA library not built: {_LIB_PATH} is missing; run "
                "`python -c 'import __graft_entry__ as g; g.build()'` first")
        lib = ctypes.CDLL(_LIB_PATH)
        P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        PP = ctypes.POINTER(ctypes.c_void_p)
        lib.ar_add_rmsnorm.restype = i32
        lib.ar_add_rmsnorm.argtypes = [PP, P, P, P, P, i64, i64, i32, f32, i32, i32, P]
        lib.ar_add_rmsnorm_quant_fp8_group.restype = i32
        lib.ar_add_rmsnorm_quant_fp8_group.argtypes = [PP, P, P, P, P, P, P, i64, i64, i32, i32,
                                                       f32, i32, i32, P]
        lib.ar_add_rmsnorm_quant_fp8_group_strided.restype = i32
        lib.ar_add_rmsnorm_quant_fp8_group_strided.argtypes = [PP, P, P, P, P, i64, i64, P, P, i64,
                                                               i64, i32, i32, f32, i32, i32, P]
        lib.qk_norm_sharded.restype = i32
        lib.qk_norm_sharded.argtypes = [PP, P, P, PP, PP, i64, i64, i64, i32, f32, i32, P]
        lib.ar_plan_query.restype = i32
        lib.ar_plan_query.argtypes = [i32, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_int)]
        lib.ar_plan_load.restype = i32
        lib.ar_plan_load.argtypes = [ctypes.c_char_p]
        lib.ar_plan_force.restype = i32
        lib.ar_plan_force.argtypes = [i32, i32]
        lib.ar_plan_table_size.restype = i32
        lib.ar_plan_table_size.argtypes = []
        lib.ar_status_string.restype = ctypes.c_char_p
        lib.ar_status_string.argtypes = [i32]
        lib.ar_device_status.restype = i32
        lib.ar_device_status.argtypes = [i32]
        lib.ar_test_withhold_row.restype = i32
        lib.ar_test_withhold_row.argtypes = [i64]
        if os.path.exists(_PLAN_TABLE):
            st = lib.ar_plan_load(_PLAN_TABLE.encode())
            if st != 0:
                raise RuntimeError(f"shipped plan table {_PLAN_TABLE} rejected (status {st})")
        _lib = lib
        return lib


def ar_status_string(status: int) -> str:
    return load_library().ar_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise ARError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    sdev = getattr(stream, "device", None)
    if sdev is not None and torch.device(sdev) != device:
        raise ValueError(f"stream belongs to {sdev}, tensors to {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float16") from None


# ----------------------------------------------------------------------------
# argument checks.  Every tensor is checked before anything is launched: a
# host pointer, a buffer on another device or a buffer shorter than the call
# implies would otherwise reach a kernel as an illegal address.  Order:
# types and dtypes, then shapes and layouts, then devices, so each mistake
# gets its own message.
# ----------------------------------------------------------------------------

def _tensor(name, t):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    return t


def _same_dtype(name, t, dtype):
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}; the call's 16-bit dtype is {dtype}")


def _rows(t: torch.Tensor, H: int, name: str = "partials[0]") -> int:
    """Token count of a [..., H] tensor: numel // H (leading dims flattened)."""
    if t.dim() < 1 or t.shape[-1] != H:
        raise ValueError(f"{name}: last dimension {tuple(t.shape)[-1:]} != hidden size {H}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.numel() // H


def _dense_like(name, t, T, H):
    """t must be a contiguous [..., H] tensor of exactly T rows."""
    if t.dim() < 1 or t.shape[-1] != H or t.numel() != T * H:
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected [..., {H}] with {T} rows")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(tensors, device=None):
    """All named tensors on one CUDA device; returns it."""
    for name, t in tensors:
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{name} is on {t.device}; every tensor must be a CUDA tensor")
        if device is None:
            device = t.device
        elif t.device != device:
            raise ValueError(f"{name} is on {t.device}, other tensors on {device}")
    return device


def _norm_args(partials, residual, weight, outs):
    """Type, dtype and shape checks shared by the norm calls; returns
    (T, H, named tensors) for the device check that comes last."""
    if not isinstance(partials, (list, tuple)) or not partials:
        raise TypeError("partials must be a non-empty list of tensors")
    if len(partials) > AR_MAX_W:
        raise ValueError(f"{len(partials)} partials; at most {AR_MAX_W}")
    _tensor("weight", weight)
    _dtype(weight)
    if weight.dim() != 1 or not weight.is_contiguous():
        raise ValueError(f"weight must be a contiguous 1-D [H] tensor, got shape {tuple(weight.shape)}")
    H = weight.shape[0]
    named = [(f"partials[{w}]", _tensor(f"partials[{w}]", p)) for w, p in enumerate(partials)]
    if residual is not None:
        named.append(("residual", _tensor("residual", residual)))
    for name, t in named:
        _same_dtype(name, t, weight.dtype)
    T = _rows(partials[0], H)
    for name, t in named:
        _dense_like(name, t, T, H)
    for name, t, dtype in outs:
        if t is None:
            continue
        _tensor(name, t)
        if dtype is not None:
            _same_dtype(name, t, dtype)
        _dense_like(name, t, T, H)
    return T, H, named + [("weight", weight)] + [(n, t) for n, t, _ in outs]


def ar_add_rmsnorm(partials, residual, weight, out, residual_out=None, eps: float = 1e-6,
                   gemma: bool = False, stream=None) -> None:
    """out = RMSNorm(residual + sum(partials)) * weight (or 1 + weight);
    residual_out = residual + sum(partials).  ``residual`` and
    ``residual_out`` may be None.  All tensors contiguous [..., H] of one
    16-bit dtype on one CUDA device; the call runs on that device."""
    if out is None:
        raise TypeError("out is required")
    T, H, named = _norm_args(partials, residual, weight,
                             [("out", out, weight.dtype), ("residual_out", residual_out, weight.dtype)])
    device = _on_device(named)
    lib = load_library()
    with torch.cuda.device(device):
        _check("ar_add_rmsnorm", lib.ar_add_rmsnorm(
            _ptrs(partials), _ptr(residual), _ptr(weight), _ptr(out), _ptr(residual_out),
            T, H, len(partials), float(eps), int(bool(gemma)), _dtype(weight),
            _stream(stream, device)))


def ar_add_rmsnorm_quant_fp8_group(partials, residual, weight, out_fp8, scales, out_y=None,
                                   residual_out=None, eps: float = 1e-6, gemma: bool = False,
                                   group: int = 128, stream=None) -> None:
    """As ar_add_rmsnorm, then per-group e4m3 codes ``out_fp8`` (uint8 or
    float8_e4m3fn [..., H]) and fp32 ``scales``; the 16-bit y goes to
    ``out_y`` when given.  ``scales`` is a [T, H/group] tensor of any strides
    (e.g. the transpose of a [H/group, T] buffer) or a contiguous
    [..., H/group] tensor."""
    for name, t in (("out_fp8", out_fp8), ("scales", scales)):
        if t is None:
            raise TypeError(f"{name} is required")
        _tensor(name, t)
    if out_fp8.element_size() != 1 or out_fp8.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"out_fp8 must be uint8 or float8_e4m3fn, got {out_fp8.dtype}")
    if scales.dtype != torch.float32:
        raise TypeError(f"scales must be float32, got {scales.dtype}")
    T, H, named = _norm_args(partials, residual, weight,
                             [("out_fp8", out_fp8, None), ("out_y", out_y, weight.dtype),
                              ("residual_out", residual_out, weight.dtype)])
    G = H // group if group > 0 else 0
    if scales.dim() == 2 and tuple(scales.shape) == (T, G):
        s_t, s_g = scales.stride()
    elif scales.is_contiguous() and scales.numel() == T * G:
        s_t, s_g = G, 1
    else:
        raise ValueError(f"scales must be [T, {G}] (any strides) or contiguous [..., {G}]")
    device = _on_device(named + [("scales", scales)])
    lib = load_library()
    with torch.cuda.device(device):
        _check("ar_add_rmsnorm_quant_fp8_group", lib.ar_add_rmsnorm_quant_fp8_group_strided(
            _ptrs(partials), _ptr(residual), _ptr(weight), _ptr(out_fp8), _ptr(scales), s_t, s_g,
            _ptr(out_y), _ptr(residual_out), T, H, len(partials), int(group), float(eps),
            int(bool(gemma)), _dtype(weight), _stream(stream, device)))


def qk_norm_sharded(qkv, q_weight, k_weight, q_out, k_out, q_size: int, kv_size: int,
                    eps: float = 1e-6, stream=None) -> None:
    """Sharded QK-norm over W = len(qkv) shards, each [T, q_size/W + 2*kv_size/W].
    q_out[w] / k_out[w] are dense [T, q_size/W] / [T, kv_size/W] tensors, or,
    for the in-place form, the views qkv[w][:, :qs] and qkv[w][:, qs:qs+ks]."""
    if not isinstance(qkv, (list, tuple)) or not qkv:
        raise TypeError("qkv must be a non-empty list of tensors")
    W = len(qkv)
    if W > AR_MAX_W:
        raise ValueError(f"{W} shards; at most {AR_MAX_W}")
    if not isinstance(q_out, (list, tuple)) or not isinstance(k_out, (list, tuple)) or \
            len(q_out) != W or len(k_out) != W:
        raise ValueError(f"q_out and k_out must be lists of {W} tensors")
    q_size, kv_size = int(q_size), int(kv_size)
    if q_size <= 0 or kv_size <= 0 or q_size % W or kv_size % W:
        raise ValueError(f"q_size {q_size} and kv_size {kv_size} must be positive multiples of W={W}")
    for name, t, n in (("q_weight", q_weight, q_size), ("k_weight", k_weight, kv_size)):
        _tensor(name, t)
        _dtype(t)
        if t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor of {n} elements, got {tuple(t.shape)}")
    _same_dtype("k_weight", k_weight, q_weight.dtype)
    qs, ks = q_size // W, kv_size // W
    row = qs + 2 * ks
    named = [("q_weight", q_weight), ("k_weight", k_weight)]
    for w in range(W):
        _tensor(f"qkv[{w}]", qkv[w])
        _same_dtype(f"qkv[{w}]", qkv[w], q_weight.dtype)
    T = _rows(qkv[0], row, "qkv[0]")
    for w in range(W):
        _dense_like(f"qkv[{w}]", qkv[w], T, row)
        named.append((f"qkv[{w}]", qkv[w]))
        for name, out, off, width in ((f"q_out[{w}]", q_out[w], 0, qs), (f"k_out[{w}]", k_out[w], qs, ks)):
            _tensor(name, out)
            _same_dtype(name, out, q_weight.dtype)
            inplace = (out.data_ptr() == qkv[w].data_ptr() + off * qkv[w].element_size()
                       and out.dim() == 2 and tuple(out.shape) == (T, width)
                       and out.stride() == (row, 1))
            if not inplace and not (out.is_contiguous() and out.numel() == T * width):
                raise ValueError(f"shard {w}: output must be a dense [T, {width}] tensor or the "
                                 f"in-place view of qkv[{w}]")
            named.append((name, out))
    device = _on_device(named)
    lib = load_library()
    with torch.cuda.device(device):
        _check("qk_norm_sharded", lib.qk_norm_sharded(
            _ptrs(qkv), _ptr(q_weight), _ptr(k_weight), _ptrs(q_out), _ptrs(k_out), T, q_size,
            kv_size, W, float(eps), _dtype(q_weight), _stream(stream, device)))


def ar_plan_query(variant: int, T: int, H: int, W: int, dtype: int) -> int:
    pid = ctypes.c_int(-1)
    _check("ar_plan_query", load_library().ar_plan_query(variant, T, H, W, dtype, ctypes.byref(pid)))
    return pid.value


def ar_plan_load(path) -> int:
    return load_library().ar_plan_load(None if path is None else str(path).encode())


def ar_plan_force(variant: int, plan_id: int) -> int:
    return load_library().ar_plan_force(variant, plan_id)


def ar_plan_table_size() -> int:
    return load_library().ar_plan_table_size()


def ar_device_status(clear: bool = True) -> int:
    """Synchronise the current device; AR_ETIMEDOUT (5) if a bounded device
    wait ran out since the last clear, else 0."""
    return load_library().ar_device_status(int(bool(clear)))


def ar_test_withhold_row(row: int) -> int:
    """Test hook: the next bulk-staged launch never issues row `row`'s copies."""
    return load_library().ar_test_withhold_row(int(row))
