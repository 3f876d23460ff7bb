"""ctypes binding of the multi-GPU form in ``include/ar_comm.h``.

``Comm``       one rank of a communicator over W processes, one GPU each.
               Creating it exchanges the ranks' handle records through
               ``torch.distributed`` (any backend) and maps every peer's
               region; its calls are collective: every rank makes the same
               calls in the same order.
``CommGroup``  W ranks inside this process on one GPU, every rank's part run
               in one cooperative launch: the same exchange protocol and
               kernels on one device (tests, single-GPU emulation).
``register``   an integer id for a ``Comm``, by which the torch operators
               ``torch.ops.ar_b200.tp_*`` and the graph rewrite's all-reduce
               marker name it (an operator schema cannot carry the object).

Argument marshalling only: tensors are checked (type, dtype, shape,
contiguity, device) before anything reaches the library, and every step of
the computation runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import binding as B

ALGOS = {"auto": 0, "oneshot": 1, "twoshot": 2}
HANDLE_BYTES = 128

_configured = False


def _lib():
    global _configured
    lib = B.load_library()
    if not _configured:
        P, i64, i32, f32, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_uint64
        PP = ctypes.POINTER(ctypes.c_void_p)
        PPc = ctypes.POINTER(ctypes.c_void_p)
        sig = {
            "ar_comm_create": [i32, i32, i64, PPc],
            "ar_comm_create_group": [i32, i64, PPc],
            "ar_comm_handle": [P, P],
            "ar_comm_check_handles": [P, i32],
            "ar_comm_open": [P, P],
            "ar_comm_destroy": [P],
            "ar_comm_set_timeout": [P, u64],
            "ar_comm_set_oneshot_max": [P, i64],
            "ar_comm_algo": [P, i64, i64, ctypes.POINTER(ctypes.c_int)],
            "ar_comm_status": [P, i32],
            "ar_comm_test_withhold": [P, i32],
            "ar_comm_allreduce_add_rmsnorm": [P, P, P, P, P, P, i64, i64, f32, i32, i32, i32, P],
            "ar_comm_allreduce_add_rmsnorm_quant_fp8_group":
                [P, P, P, P, P, P, P, P, i64, i64, i32, f32, i32, i32, i32, P],
            "ar_comm_qk_norm_sharded": [P, P, P, P, P, P, i64, i64, i64, f32, i32, P],
            "ar_group_allreduce_add_rmsnorm": [P, PP, PP, P, PP, PP, i64, i64, f32, i32, i32, i32, P],
            "ar_group_allreduce_add_rmsnorm_quant_fp8_group":
                [P, PP, PP, P, PP, PP, PP, PP, i64, i64, i32, f32, i32, i32, i32, P],
            "ar_group_qk_norm_sharded": [P, PP, P, P, PP, PP, i64, i64, i64, f32, i32, P],
        }
        for name, argtypes in sig.items():
            fn = getattr(lib, name)
            fn.restype = i32
            fn.argtypes = argtypes
        _configured = True
    return lib


def _algo(algo) -> int:
    if isinstance(algo, int):
        return algo
    try:
        return ALGOS[algo]
    except KeyError:
        raise ValueError(f"algo must be one of {list(ALGOS)}") from None


def exchange_records(record: bytes, group=None) -> bytes:
    """Every rank's handle record, concatenated in rank order (an all-gather
    over ``group``; a rank that never joins makes the others fail with the
    process group's timeout)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    records = [None] * world
    dist.all_gather_object(records, bytes(record), group=group)
    for i, r in enumerate(records):
        if not isinstance(r, (bytes, bytearray)) or len(r) != HANDLE_BYTES:
            raise RuntimeError(f"rank {i} sent a malformed handle record")
    return b"".join(records)


def oneshot_limit(rows, H: int) -> int:
    """From measured [T, one-shot us, two-shot us] rows in increasing T: the
    per-rank bytes T*H*2 of the largest T up to which one-shot was never
    slower (0 when two-shot already wins at the smallest T)."""
    limit = 0
    for T, one, two in rows:
        if one > two:
            break
        limit = T * H * 2
    return limit


def check_records(blob: bytes, world: int) -> int:
    """The library's consistency check of a gathered record set (host only):
    0 when every rank's record agrees, else an ar_status."""
    return _lib().ar_comm_check_handles(ctypes.c_char_p(blob), world)


_REGISTRY: dict = {}
_NEXT_ID = [1]


def register(c: "Comm") -> int:
    """Register a rank-form communicator; returns the id the tensor-parallel
    operators and ``fx_patterns.tp_all_reduce_reference`` take.  Every rank
    registers its own communicator; ids are per process (ranks registering
    in the same order get the same ids).  Valid until ``unregister``."""
    if not isinstance(c, Comm):
        raise TypeError("only a rank-form Comm can be registered")
    i = _NEXT_ID[0]
    _NEXT_ID[0] += 1
    _REGISTRY[i] = c
    return i


def unregister(comm_id: int) -> None:
    _REGISTRY.pop(int(comm_id), None)


def lookup(comm_id: int):
    c = _REGISTRY.get(int(comm_id))
    if c is None:
        raise ValueError(f"no communicator is registered as {comm_id}")
    return c


class _Base:
    _c = None

    def set_timeout(self, seconds: float) -> None:
        B._check("ar_comm_set_timeout", _lib().ar_comm_set_timeout(self._c, int(seconds * 1e9)))

    def set_oneshot_max(self, nbytes: int) -> None:
        B._check("ar_comm_set_oneshot_max", _lib().ar_comm_set_oneshot_max(self._c, int(nbytes)))

    def algo(self, T: int, H: int) -> str:
        out = ctypes.c_int(-1)
        B._check("ar_comm_algo", _lib().ar_comm_algo(self._c, T, H, ctypes.byref(out)))
        return {v: k for k, v in ALGOS.items()}[out.value]

    def status(self, clear: bool = True) -> int:
        """Synchronises; 5 (AR_ETIMEDOUT) if a cross-rank wait ran out."""
        return _lib().ar_comm_status(self._c, int(bool(clear)))

    def test_withhold(self, rank: int) -> None:
        B._check("ar_comm_test_withhold", _lib().ar_comm_test_withhold(self._c, int(rank)))

    def close(self) -> None:
        """Free this communicator.  For a multi-process communicator every
        rank must be done with its calls first (a rank's region may still be
        read by another rank's last kernel): synchronise and meet the other
        ranks (e.g. a torch.distributed barrier) before closing."""
        if self._c is not None:
            c, self._c = self._c, None
            B._check("ar_comm_destroy", _lib().ar_comm_destroy(c))

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _norm_checks(named_parts, named_res, weight, named_outs):
    """Shapes and dtypes of one rank's tensors; returns (T, H, named list)."""
    B._tensor("weight", weight)
    B._dtype(weight)
    if weight.dim() != 1 or not weight.is_contiguous():
        raise ValueError(f"weight must be a contiguous 1-D [H] tensor, got {tuple(weight.shape)}")
    H = weight.shape[0]
    name0, p0 = named_parts[0]
    B._tensor(name0, p0)
    B._same_dtype(name0, p0, weight.dtype)
    T = B._rows(p0, H, name0)
    named = [("weight", weight)]
    for name, t in list(named_parts) + list(named_res):
        if t is None:
            continue
        B._tensor(name, t)
        B._same_dtype(name, t, weight.dtype)
        B._dense_like(name, t, T, H)
        named.append((name, t))
    for name, t, dtype in named_outs:
        if t is None:
            continue
        B._tensor(name, t)
        if dtype is not None:
            B._same_dtype(name, t, dtype)
        B._dense_like(name, t, T, H)
        named.append((name, t))
    return T, H, named


def _fp8_checks(name_q, q, name_s, s, T, H, group):
    for name, t in ((name_q, q), (name_s, s)):
        if t is None:
            raise TypeError(f"{name} is required")
        B._tensor(name, t)
    if q.element_size() != 1 or q.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name_q} must be uint8 or float8_e4m3fn, got {q.dtype}")
    if s.dtype != torch.float32:
        raise TypeError(f"{name_s} must be float32, got {s.dtype}")
    G = H // group
    if not s.is_contiguous() or s.numel() != T * G:
        raise ValueError(f"{name_s} must be a contiguous [T, {G}] tensor")


def _qk_checks(qkv, q_weight, k_weight, q_out, k_out, q_size, kv_size, W, idx=""):
    """Shapes of one rank's QK tensors; returns (T, in_place, named list)."""
    for name, t, n in (("q_weight", q_weight, q_size), ("k_weight", k_weight, kv_size)):
        B._tensor(name, t)
        B._dtype(t)
        if t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor of {n} elements")
    B._same_dtype("k_weight", k_weight, q_weight.dtype)
    if q_size % W or kv_size % W:
        raise ValueError(f"q_size and kv_size must be multiples of W={W}")
    qs, ks = q_size // W, kv_size // W
    row = qs + 2 * ks
    B._tensor(f"qkv{idx}", qkv)
    B._same_dtype(f"qkv{idx}", qkv, q_weight.dtype)
    T = B._rows(qkv, row, f"qkv{idx}")
    named = [("q_weight", q_weight), ("k_weight", k_weight), (f"qkv{idx}", qkv)]
    inplace = []
    for name, out, off, width in ((f"q_out{idx}", q_out, 0, qs), (f"k_out{idx}", k_out, qs, ks)):
        B._tensor(name, out)
        B._same_dtype(name, out, q_weight.dtype)
        ip = (out.data_ptr() == qkv.data_ptr() + off * qkv.element_size() and out.dim() == 2
              and tuple(out.shape) == (T, width) and out.stride() == (row, 1))
        if not ip and not (out.is_contiguous() and out.numel() == T * width):
            raise ValueError(f"{name} must be a dense [T, {width}] tensor or the in-place view of qkv")
        inplace.append(ip)
        named.append((name, out))
    return T, inplace, named


class Comm(_Base):
    """This rank of a W-rank communicator (one process per GPU).

    ``max_elems`` bounds T * H of every call.  ``group`` is a
    torch.distributed process group (default: the world; without an
    initialised process group, a single rank); the handle records are
    exchanged over it at construction."""

    def __init__(self, max_elems: int, group=None, device=None):
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            self.rank = dist.get_rank(group)
            self.world = dist.get_world_size(group)
        elif group is None:
            self.rank, self.world = 0, 1      # no process group: a single rank
        else:
            raise RuntimeError("a process group was given but torch.distributed is not initialised")
        self.group = group
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        lib = _lib()
        c = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            B._check("ar_comm_create", lib.ar_comm_create(self.rank, self.world, int(max_elems),
                                                          ctypes.byref(c)))
        self._c = c
        if self.world > 1:
            rec = ctypes.create_string_buffer(HANDLE_BYTES)
            B._check("ar_comm_handle", lib.ar_comm_handle(self._c, rec))
            blob = exchange_records(rec.raw, group)
            B._check("ar_comm_check_handles", lib.ar_comm_check_handles(ctypes.c_char_p(blob), self.world))
            B._check("ar_comm_open", lib.ar_comm_open(self._c, ctypes.c_char_p(blob)))

    def _run(self, fn, *args, stream=None):
        with torch.cuda.device(self.device):
            B._check(fn, getattr(_lib(), fn)(self._c, *args, B._stream(stream, self.device)))

    def _device(self, named):
        dev = B._on_device(named)
        if dev != self.device:
            raise ValueError(f"tensors are on {dev}; the communicator is on {self.device}")

    def allreduce_add_rmsnorm(self, partial, residual, weight, out, residual_out=None,
                              eps: float = 1e-6, gemma: bool = False, algo="auto", stream=None):
        """out = RMSNorm(residual + sum over ranks of partial) (Gemma: * (1 + w));
        residual_out = residual + sum over ranks of partial.  Collective."""
        if out is None:
            raise TypeError("out is required")
        T, H, named = _norm_checks([("partial", partial)], [("residual", residual)], weight,
                                   [("out", out, weight.dtype), ("residual_out", residual_out, weight.dtype)])
        self._device(named)
        self._run("ar_comm_allreduce_add_rmsnorm", B._ptr(partial), B._ptr(residual), B._ptr(weight),
                  B._ptr(out), B._ptr(residual_out), T, H, float(eps), int(bool(gemma)),
                  B._dtype(weight), _algo(algo), stream=stream)

    def allreduce_add_rmsnorm_quant_fp8_group(self, partial, residual, weight, out_fp8, scales,
                                              out_y=None, residual_out=None, eps: float = 1e-6,
                                              gemma: bool = False, algo="auto", stream=None):
        """As allreduce_add_rmsnorm, then per-group (128) e4m3 codes and fp32
        row-major [T, H/128] scales.  Collective."""
        T, H, named = _norm_checks([("partial", partial)], [("residual", residual)], weight,
                                   [("out_fp8", out_fp8, None), ("out_y", out_y, weight.dtype),
                                    ("residual_out", residual_out, weight.dtype)])
        _fp8_checks("out_fp8", out_fp8, "scales", scales, T, H, 128)
        self._device(named + [("scales", scales)])
        self._run("ar_comm_allreduce_add_rmsnorm_quant_fp8_group", B._ptr(partial), B._ptr(residual),
                  B._ptr(weight), B._ptr(out_fp8), B._ptr(scales), B._ptr(out_y),
                  B._ptr(residual_out), T, H, 128, float(eps), int(bool(gemma)), B._dtype(weight),
                  _algo(algo), stream=stream)

    def tune_oneshot_max(self, H: int = 8192, Ts=(1, 2, 4, 8, 16, 32, 64, 128, 256, 512),
                         iters: int = 50, group=None) -> int:
        """Measure the one-shot / two-shot crossover on these ranks and set it.

        Collective: every rank calls it with the same arguments.  For each T
        both forms run `iters` times (bf16, [T, H], CUDA events on the current
        stream, the max over ranks as the time); the largest per-rank size
        T*H*2 up to which one-shot was faster for every measured T below it
        becomes ``set_oneshot_max``.  Returns that byte count; the times are
        kept in ``self.crossover_us`` as [T, one-shot us, two-shot us]."""
        import torch.distributed as dist
        dev = self.device
        use_dist = dist.is_available() and dist.is_initialized() and self.world > 1
        Tmax = max(Ts)
        g = torch.Generator(device=dev).manual_seed(1234)
        part = torch.randn(Tmax, H, generator=g, device=dev).to(torch.bfloat16)
        res = torch.randn(Tmax, H, generator=g, device=dev).to(torch.bfloat16)
        w = torch.ones(H, dtype=torch.bfloat16, device=dev)
        out = torch.empty_like(part)
        stream = torch.cuda.current_stream(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rows = []
        for T in sorted(Ts):
            us = []
            for algo in ("oneshot", "twoshot"):
                call = lambda: self.allreduce_add_rmsnorm(part[:T], res[:T], w, out[:T], None,
                                                          algo=algo, stream=stream)
                for _ in range(5):
                    call()
                torch.cuda.synchronize(dev)
                if use_dist:
                    dist.barrier(group=group)
                a.record(stream)
                for _ in range(iters):
                    call()
                b.record(stream)
                b.synchronize()
                t = torch.tensor([a.elapsed_time(b) * 1e3 / iters], dtype=torch.float64, device=dev)
                if use_dist:
                    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
                us.append(float(t.item()))
            rows.append([T, round(us[0], 3), round(us[1], 3)])
        limit = oneshot_limit(rows, H)
        self.crossover_us = rows
        self.set_oneshot_max(limit)
        return limit

    def qk_norm_sharded(self, qkv, q_weight, k_weight, q_out, k_out, q_size: int, kv_size: int,
                        eps: float = 1e-6, stream=None):
        """This rank's shard of the sharded QK-norm (q and k normalised over
        the full width; only the per-token sums of squares cross ranks)."""
        T, _, named = _qk_checks(qkv, q_weight, k_weight, q_out, k_out, int(q_size), int(kv_size),
                                 self.world)
        self._device(named)
        self._run("ar_comm_qk_norm_sharded", B._ptr(qkv), B._ptr(q_weight), B._ptr(k_weight),
                  B._ptr(q_out), B._ptr(k_out), T, int(q_size), int(kv_size), float(eps),
                  B._dtype(q_weight), stream=stream)


class CommGroup(_Base):
    """W ranks in this process on one GPU; each call runs every rank's part
    in one cooperative launch.  Per-rank arguments are lists of W tensors."""

    def __init__(self, world: int, max_elems: int, device=None):
        self.world = int(world)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        c = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            B._check("ar_comm_create_group", _lib().ar_comm_create_group(self.world, int(max_elems),
                                                                         ctypes.byref(c)))
        self._c = c

    def _lists(self, **kw):
        for name, v in kw.items():
            if v is None:
                continue
            if not isinstance(v, (list, tuple)) or len(v) != self.world:
                raise ValueError(f"{name} must be a list of {self.world} tensors")

    def _run(self, fn, *args, stream=None):
        with torch.cuda.device(self.device):
            B._check(fn, getattr(_lib(), fn)(self._c, *args, B._stream(stream, self.device)))

    def _device(self, named):
        dev = B._on_device(named)
        if dev != self.device:
            raise ValueError(f"tensors are on {dev}; the group is on {self.device}")

    @staticmethod
    def _arr(ts):
        return None if ts is None else (ctypes.c_void_p * len(ts))(
            *[None if t is None else t.data_ptr() for t in ts])

    def allreduce_add_rmsnorm(self, partials, residuals, weight, outs, residual_outs=None,
                              eps: float = 1e-6, gemma: bool = False, algo="auto", stream=None):
        self._lists(partials=partials, residuals=residuals, outs=outs, residual_outs=residual_outs)
        named_all = []
        T = H = None
        for r in range(self.world):
            t, h, named = _norm_checks(
                [(f"partials[{r}]", partials[r])],
                [(f"residuals[{r}]", residuals[r] if residuals else None)], weight,
                [(f"outs[{r}]", outs[r], weight.dtype),
                 (f"residual_outs[{r}]", residual_outs[r] if residual_outs else None, weight.dtype)])
            if T is not None and (t, h) != (T, H):
                raise ValueError(f"rank {r}'s tensors have {t} rows; rank 0's {T}")
            T, H = t, h
            named_all += named
        self._device(named_all)
        self._run("ar_group_allreduce_add_rmsnorm", self._arr(partials), self._arr(residuals),
                  B._ptr(weight), self._arr(outs), self._arr(residual_outs), T, H, float(eps),
                  int(bool(gemma)), B._dtype(weight), _algo(algo), stream=stream)

    def allreduce_add_rmsnorm_quant_fp8_group(self, partials, residuals, weight, out_fp8s, scales,
                                              out_ys=None, residual_outs=None, eps: float = 1e-6,
                                              gemma: bool = False, algo="auto", stream=None):
        self._lists(partials=partials, residuals=residuals, out_fp8s=out_fp8s, scales=scales,
                    out_ys=out_ys, residual_outs=residual_outs)
        named_all = []
        T = H = None
        for r in range(self.world):
            t, h, named = _norm_checks(
                [(f"partials[{r}]", partials[r])],
                [(f"residuals[{r}]", residuals[r] if residuals else None)], weight,
                [(f"out_fp8s[{r}]", out_fp8s[r], None),
                 (f"out_ys[{r}]", out_ys[r] if out_ys else None, weight.dtype),
                 (f"residual_outs[{r}]", residual_outs[r] if residual_outs else None, weight.dtype)])
            if T is not None and (t, h) != (T, H):
                raise ValueError(f"rank {r}'s tensors have {t} rows; rank 0's {T}")
            T, H = t, h
            _fp8_checks(f"out_fp8s[{r}]", out_fp8s[r], f"scales[{r}]", scales[r], T, H, 128)
            named_all += named + [(f"scales[{r}]", scales[r])]
        self._device(named_all)
        self._run("ar_group_allreduce_add_rmsnorm_quant_fp8_group", self._arr(partials),
                  self._arr(residuals), B._ptr(weight), self._arr(out_fp8s), self._arr(scales),
                  self._arr(out_ys), self._arr(residual_outs), T, H, 128, float(eps),
                  int(bool(gemma)), B._dtype(weight), _algo(algo), stream=stream)

    def qk_norm_sharded(self, qkv, q_weight, k_weight, q_outs, k_outs, q_size: int, kv_size: int,
                        eps: float = 1e-6, stream=None):
        self._lists(qkv=qkv, q_outs=q_outs, k_outs=k_outs)
        named_all, T, modes = [], None, set()
        for r in range(self.world):
            t, ip, named = _qk_checks(qkv[r], q_weight, k_weight, q_outs[r], k_outs[r], int(q_size),
                                      int(kv_size), self.world, f"[{r}]")
            if T is not None and t != T:
                raise ValueError(f"rank {r}'s shard has {t} tokens; rank 0's {T}")
            T = t
            modes.add(tuple(ip))
            named_all += named
        if len(modes) != 1 or len(set(next(iter(modes)))) != 1:
            raise ValueError("outputs must be all dense or all the in-place views of qkv")
        self._device(named_all)
        self._run("ar_group_qk_norm_sharded", self._arr(qkv), B._ptr(q_weight), B._ptr(k_weight),
                  self._arr(q_outs), self._arr(k_outs), T, int(q_size), int(kv_size), float(eps),
                  B._dtype(q_weight), stream=stream)
