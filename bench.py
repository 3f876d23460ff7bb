"""Benchmark of the fused W-way reduce + residual add + RMSNorm library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|decode|tiny|fp8|qk] [--no-sweep]
    python bench.py --sweep-only --sweep qk [--sweep-T 1 64 2048 ...] [--force-plan P]
    python bench.py --sweep-only --sweep exchange   # the exchange kernels at world size 1

One step = one pass over every call of the chosen workload, each call
through the C ABI, the whole step captured once in a CUDA graph per rotating
buffer set and replayed.  The default workload is the largest single-GPU
configuration of the fused reduce + add + RMSNorm: prefill, dead residual,
T=8192, H=4096, W=8 bf16 partials (671 MB of algorithmic traffic per call,
inputs larger than L2).  Buffer sets rotate so the data a step touches was
last touched more than 2x L2 ago (cold HBM), or the inputs alone exceed L2.
Rank 0 prints one JSON line, last; the per-call sweep of every workload is
printed as plain text lines before it.

value       achieved GB/s = algorithmic bytes of all ranks' steps / max-over-ranks
            device time (CUDA events around exactly K steps)
e2e         the same metric through the same public call with host buffers:
            pinned host -> device copies of every input, the call, and the
            device -> host copy of every output, all inside the timed region
roofline    the step's kernel against the measured HBM copy bandwidth
cpu_baseline / --impl reference
            the fp64 CPU oracle on the host cores (threads over row blocks),
            on a bounded sample of the same workload (rank 0, N = 1)
sweep       per-call microseconds and GB/s of every workload (not timed in
            the headline number); summarised in the JSON line
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "µs/call and achieved HBM GB/s (% of ~8 TB/s) for fused W-reduce+add+RMSNorm"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


# ----------------------------------------------------------------------------
# workloads as lists of calls
# ----------------------------------------------------------------------------

def workload_calls(name: str, Ts=None):
    """Every call of a workload: (kind, workload, T, dtype), over the
    workload's token counts or the given ones."""
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    if name in ("tiny", "decode", "prefill", "fp8"):
        w = wl.WORKLOADS[name]
        return [("norm", w, T, dt) for dt in w.dtypes for T in (Ts or w.Ts)]
    if name == "qk":
        return [("qk", wl.QK, T, "bf16") for T in (Ts or wl.QK.Ts)]
    raise ValueError(name)


def call_bytes(call) -> int:
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    kind, w, T, dt = call
    if kind == "qk":
        return wl.qk_bytes(T, w.W, w.q_size, w.kv_size)
    return wl.norm_bytes(T, w.H, w.W, w.residual is not None, w.write_residual, fp8=w.fp8)


def describe(name: str) -> str:
    return {
        "decode": "decode window: T in {1,2,4,8,16,32,64,80} x {bf16,fp16}, H=8192, W=4 partials "
                  "N(0,0.5), residual N(0,1), Gemma weight N(0,0.1), eps=1e-6, y + residual_out",
        "tiny": "tiny: T=16, H=4096, W=2 bf16, standard RMSNorm, y + residual_out",
        "prefill": "prefill dead-residual: T=8192, H=4096, W=8 bf16 partials N(0,1/8), eps=1e-5, y only",
        "fp8": "per-group FP8: T=1..32768 (powers of 2), H=5120, W=4 bf16, group 128 e4m3 + y + residual_out",
        "qk": "sharded QK-norm: T in {1,64,2048}, W=8, q_size=6144, kv_size=1024 bf16",
    }[name]


class CallBuffers:
    """Device inputs and outputs of one call (one buffer set)."""

    def __init__(self, call, device, seed_offset=0, inputs=None):
        import torch
        from tensor_allreduce_residual_ar_b200 import workloads as wl
        kind, w, T, dt = call
        self.call = call
        td = {"bf16": torch.bfloat16, "fp16": torch.float16}[dt]
        if kind == "qk":
            inp = inputs or wl.make_qk_inputs(w, T, dt, device=device,
                                              seed=wl.seed_for("qk", T) + seed_offset)
            self.inp = inp
            self.qkv = [x.clone() for x in inp.qkv]
            self.qw, self.kw = inp.q_weight.clone(), inp.k_weight.clone()
            qs, ks = w.q_size // w.W, w.kv_size // w.W
            self.q_out = [torch.empty((T, qs), dtype=td, device=device) for _ in range(w.W)]
            self.k_out = [torch.empty((T, ks), dtype=td, device=device) for _ in range(w.W)]
        else:
            inp = inputs or wl.make_norm_inputs(w, T, dt, device=device,
                                                seed=wl.seed_for(w.name, T) + seed_offset)
            self.inp = inp
            self.parts = [p.clone() for p in inp.partials]
            self.res = inp.residual.clone() if inp.residual is not None else None
            self.w = inp.weight.clone()
            self.out = torch.empty((T, w.H), dtype=td, device=device)
            self.rout = torch.empty((T, w.H), dtype=td, device=device) if w.write_residual else None
            if w.fp8:
                self.q = torch.empty((T, w.H), dtype=torch.uint8, device=device)
                self.s = torch.empty((T, w.H // w.group), dtype=torch.float32, device=device)

    def inputs(self):
        if self.call[0] == "qk":
            return self.qkv + [self.qw, self.kw]
        return self.parts + ([self.res] if self.res is not None else []) + [self.w]

    def outputs(self):
        if self.call[0] == "qk":
            return self.q_out + self.k_out
        w = self.call[1]
        outs = [self.out] + ([self.rout] if self.rout is not None else [])
        if w.fp8:
            outs += [self.q, self.s]
        return outs

    def run(self, ar):
        kind, w, T, dt = self.call
        if kind == "qk":
            ar.qk_norm_sharded(self.qkv, self.qw, self.kw, self.q_out, self.k_out, w.q_size,
                               w.kv_size, eps=self.inp.eps)
        elif w.fp8:
            ar.ar_add_rmsnorm_quant_fp8_group(self.parts, self.res, self.w, self.q, self.s, self.out,
                                              self.rout, eps=self.inp.eps, gemma=w.gemma)
        else:
            ar.ar_add_rmsnorm(self.parts, self.res, self.w, self.out, self.rout, eps=self.inp.eps,
                              gemma=w.gemma)


def rotation_sets(step_bytes: int) -> int:
    """Buffer sets so a set is reused only after > 2x L2 of other traffic."""
    if step_bytes >= 4 * L2_BYTES:
        return 1
    return int(2 * L2_BYTES // step_bytes) + 2


# ----------------------------------------------------------------------------
# clocks (NVML, read-only) during the timed region
# ----------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.mem_samples = []
        self.power_w = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: clocks reported as unavailable
            self._nv = None
            self.error = str(e)

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self._h))
            except Exception:
                pass
            try:   # context for a number taken under the power cap (read-only)
                self.mem_samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_MEM))
                self.power_w.append(nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        if self._nv is None:
            return {"unavailable": getattr(self, "error", "no NVML")}
        names = [n for b, n in _REASONS.items() if self.reasons & b and b != 0x1]
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": names}
        if self.mem_samples:
            out["mem_mhz"] = statistics.median(self.mem_samples)
        if self.power_w:
            out["power_w"] = round(statistics.median(self.power_w), 1)
        return out


# ----------------------------------------------------------------------------
# multi-rank plumbing (also exercised on CPU with gloo in the tests)
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the default process group (identity
    when no group is initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def weak_scaling_value(bytes_per_rank_step: int, world: int, steps: int, max_seconds: float) -> float:
    """Whole-job GB/s: every rank processes its own calls (no data-path
    collective), so the job moves world x the per-rank bytes."""
    return world * bytes_per_rank_step * steps / max_seconds / 1e9


# ----------------------------------------------------------------------------
# measurement pieces
# ----------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C/C++ source without its comments and with whitespace runs collapsed
    (string and character literals kept), so that editing a comment does not
    count as a change of the kernels."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of what decides the timed kernels: the CUDA and host sources
    (code only) and the plan table."""
    h = hashlib.sha256()
    for rel in ("tensor_allreduce_residual_ar_b200/csrc/kernels.cuh",
                "tensor_allreduce_residual_ar_b200/csrc/ar_rmsnorm.cu",
                "tensor_allreduce_residual_ar_b200/csrc/plan.cpp",
                "tensor_allreduce_residual_ar_b200/plan_table.json"):
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            with open(p, encoding="utf-8") as f:
                text = f.read()
            h.update((text if rel.endswith(".json") else _code_only(text)).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per step from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    src, vals = None, {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line.startswith("# kernel-source-hash:"):
                src = line.split(":", 1)[1].strip()
            elif line and not line.startswith("#"):
                k, v = line.split()[:2]
                vals[k] = float(v)
    if src != kernel_source_hash():
        return None
    return vals.get(f"{workload}_dram_bytes_per_step")


def capture_step_graphs(ar, sets, stream):
    """One CUDA graph per buffer set, each holding every call of a step."""
    import torch
    graphs = []
    for bufs in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for b in bufs:
                    b.run(ar)
        graphs.append(g)
    return graphs


def time_graphs(graphs, n, stream, label=None):
    """Replay n steps; the timed region carries an NVTX range `label` so a
    profiler can restrict itself to it."""
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if label:
        torch.cuda.nvtx.range_push(label)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(n):
            graphs[i % len(graphs)].replay()
        end.record(stream)
    end.synchronize()
    if label:
        torch.cuda.nvtx.range_pop()
    return start.elapsed_time(end) / 1e3


def per_call_sweep(ar, device, stream, names, reps=20, Ts=None):
    """Per-call device time of every (workload, T, dtype): one graph holding
    the call once per rotating buffer set, replayed `reps` times."""
    import torch
    out = {}
    peak, _ = load_peaks()
    for name in names:
        rows = []
        for call in workload_calls(name, Ts):
            nbytes = call_bytes(call)
            R = min(rotation_sets(nbytes), 2048)
            base = CallBuffers(call, device)
            sets = [base] + [CallBuffers(call, device, inputs=base.inp) for _ in range(R - 1)]
            with torch.cuda.stream(stream):
                for b in sets:
                    b.run(ar)
            torch.cuda.synchronize()
            graphs = capture_step_graphs(ar, [sets], stream)
            time_graphs(graphs, 2, stream)
            sec = time_graphs(graphs, reps, stream) / (reps * R)
            row = {"T": call[2], "dtype": call[3], "us": round(sec * 1e6, 3),
                   "GBps": round(nbytes / sec / 1e9, 1),
                   "frac_of_peak": round(nbytes / sec / 1e9 / peak, 4),
                   "frac_of_8TBps": round(nbytes / sec / 1e9 / NOMINAL_HBM_GBS, 4),
                   "bytes": nbytes, "plan": plan_of(ar, call), "sets": R}
            if name in ("decode", "tiny"):
                # the same call 64 times on one buffer set: inputs L2-resident
                # (a latency figure, not a bandwidth one)
                hot = capture_step_graphs(ar, [[base] * 64], stream)
                time_graphs(hot, 2, stream)
                row["us_hot_l2"] = round(time_graphs(hot, reps, stream) / (reps * 64) * 1e6, 3)
                del hot
            rows.append(row)
            del graphs, sets, base
            torch.cuda.empty_cache()
        out[name] = rows
    return out


def plan_of(ar, call):
    kind, w, T, dt = call
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    if kind == "qk":
        return ar.ar_plan_query(2, T, w.q_size + w.kv_size, w.W, wl.DTYPE_CODE[dt])
    return ar.ar_plan_query(1 if w.fp8 else 0, T, w.H, w.W, wl.DTYPE_CODE[dt])


_E2E_IN = {"qk": ("qkv", "qw", "kw"), "norm": ("parts", "res", "w")}
_E2E_OUT = {"qk": ("q_out", "k_out"), "norm": ("out", "rout", "q", "s")}


def _carve_into(b, names, slab, off):
    """Replace b's tensors `names` by views of `slab` from byte `off` on
    (256-byte aligned each, contents copied); returns the next offset."""
    for name in names:
        v = getattr(b, name, None)
        if v is None:
            continue
        ts = v if isinstance(v, list) else [v]
        views = []
        for t in ts:
            nb = t.numel() * t.element_size()
            view = slab[off:off + nb].view(t.dtype).view(t.shape)
            view.copy_(t)
            views.append(view)
            off += (nb + 255) // 256 * 256
        setattr(b, name, views if isinstance(v, list) else views[0])
    return off


def _e2e_sizes(b):
    kind = "qk" if b.call[0] == "qk" else "norm"
    def size(names, padded):
        n = 0
        for name in names:
            v = getattr(b, name, None)
            for t in ([] if v is None else v if isinstance(v, list) else [v]):
                nb = t.numel() * t.element_size()
                n += (nb + 255) // 256 * 256 if padded else nb
        return n
    return kind, size(_E2E_IN[kind], True), size(_E2E_OUT[kind], True), \
        size(_E2E_IN[kind], False), size(_E2E_OUT[kind], False)


def e2e_measure(ar, device, stream, calls, steps):
    """End to end through the public calls with host buffers.  Every step
    copies all of its inputs from pinned host memory (one contiguous staging
    area, one host-to-device copy) and reads all of its results back into
    pinned host memory (one device-to-host copy).  Two device buffer sets
    alternate, so that step k+1's input copy and step k's result copy run on
    the two copy engines while step k computes (copy-in, compute and
    copy-out streams ordered by events).  Returns (seconds for `steps`
    steps, input bytes per step, output bytes per step)."""
    import torch
    sets = []
    for _ in range(2):
        bufs = [CallBuffers(call, device) for call in calls]
        sizes = [_e2e_sizes(b) for b in bufs]
        in_bytes = sum(x[1] for x in sizes)
        out_bytes = sum(x[2] for x in sizes)
        din = torch.empty(in_bytes, dtype=torch.uint8, device=device)
        dout = torch.empty(out_bytes, dtype=torch.uint8, device=device)
        oi = oo = 0
        for b, (kind, _, _, _, _) in zip(bufs, sizes):
            oi = _carve_into(b, _E2E_IN[kind], din, oi)
            oo = _carve_into(b, _E2E_OUT[kind], dout, oo)
        sets.append((bufs, din, dout))
    h2d = sum(_e2e_sizes(b)[3] for b in sets[0][0])
    d2h = sum(_e2e_sizes(b)[4] for b in sets[0][0])
    host_in = sets[0][1].cpu().pin_memory()
    host_out = torch.empty(sets[0][2].numel(), dtype=torch.uint8, pin_memory=True)
    torch.cuda.synchronize()

    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    computed = [ev(), ev()]
    copied_out = [ev(), ev()]
    ready = [ev(), ev()]
    for e in computed + copied_out:
        e.record(stream)

    def one_step(k):
        bufs, din, dout = sets[k & 1]
        s_in.wait_event(computed[k & 1])             # step k-2 is done with these inputs
        with torch.cuda.stream(s_in):
            din.copy_(host_in, non_blocking=True)
        ready[k & 1].record(s_in)
        stream.wait_event(ready[k & 1])
        stream.wait_event(copied_out[k & 1])         # step k-2's results have left
        with torch.cuda.stream(stream):
            for b in bufs:
                b.run(ar)
        computed[k & 1].record(stream)
        s_out.wait_event(computed[k & 1])
        with torch.cuda.stream(s_out):
            host_out.copy_(dout, non_blocking=True)
        copied_out[k & 1].record(s_out)

    for k in range(2):
        one_step(k)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for k in range(steps):
        one_step(k)
    end.record(s_out)
    s_in.wait_stream(s_out)
    end.synchronize()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3, h2d, d2h


def host_cpu():
    """Host CPU model and the number of cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": n}


def oracle_sample(calls, budget_s: float, max_steps: int | None = None, row_fraction: float = 1.0,
                  threads: int = 1):
    """Time the fp64 CPU oracle (as it stands) on steps of the workload until
    the budget is used or max_steps are done.  A step is every call of the
    workload, each on its first ceil(row_fraction * T) rows; with threads > 1
    the rows of each call are split into that many blocks, each computed by
    one oracle call on its own thread (the oracle's C entry points release
    the interpreter lock).  Returns (seconds, steps, algorithmic bytes per
    step actually processed)."""
    import math as _m
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    prepared = []
    step_bytes = 0
    for call in calls:
        kind, w, T, dt = call
        rows = max(1, int(_m.ceil(row_fraction * T)))
        if kind == "qk":
            inp = wl.make_qk_inputs(w, T, dt)
            prepared.append(("qk", inp, rows, [wl.bits(x)[:rows] for x in inp.qkv]))
            step_bytes += wl.qk_bytes(rows, w.W, w.q_size, w.kv_size)
        else:
            inp = wl.make_norm_inputs(w, T, dt)
            res = wl.bits(inp.residual)[:rows] if inp.residual is not None else None
            prepared.append(("norm", inp, rows, ([wl.bits(p)[:rows] for p in inp.partials], res)))
            step_bytes += wl.norm_bytes(rows, w.H, w.W, w.residual is not None, w.write_residual,
                                        fp8=w.fp8)
    fp8 = {id(inp): call[1].fp8 for call, (_, inp, _, _) in zip(calls, prepared)}

    def block(kind, inp, arrs, a, b):
        if kind == "qk":
            oracle.qk_norm_sharded([x[a:b] for x in arrs], wl.bits(inp.q_weight),
                                   wl.bits(inp.k_weight), inp.q_size, inp.kv_size, inp.eps,
                                   wl.DTYPE_CODE[inp.dtype])
            return
        parts, res = arrs
        o = oracle.ar_add_rmsnorm([p[a:b] for p in parts], None if res is None else res[a:b],
                                  wl.bits(inp.weight), inp.eps, inp.gemma, wl.DTYPE_CODE[inp.dtype])
        oracle.round16(o["y"], wl.DTYPE_CODE[inp.dtype])
        if inp.write_residual:
            oracle.round16(o["r"], wl.DTYPE_CODE[inp.dtype])
        if fp8[id(inp)]:
            oracle.quant_fp8_group(o["y"])

    pool = ThreadPoolExecutor(threads) if threads > 1 else None

    def one_step():
        for kind, inp, rows, arrs in prepared:
            if pool is None:
                block(kind, inp, arrs, 0, rows)
                continue
            n = min(threads, rows)
            cuts = [rows * i // n for i in range(n + 1)]
            list(pool.map(lambda i: block(kind, inp, arrs, cuts[i], cuts[i + 1]), range(n)))
    try:
        one_step()   # warm (builds the oracle library, page-faults the arrays)
        t0 = time.perf_counter()
        n = 0
        while True:
            one_step()
            n += 1
            el = time.perf_counter() - t0
            if el >= budget_s or (max_steps is not None and n >= max_steps):
                break
    finally:
        if pool is not None:
            pool.shutdown()
    return el, n, step_bytes


# ----------------------------------------------------------------------------
# multi-GPU form (N > 1): the fused exchange kernels against NCCL
# ----------------------------------------------------------------------------

TP_SHAPES = ((1, 8192), (8, 8192), (32, 8192), (80, 8192), (256, 8192), (1024, 8192), (8192, 4096))
TP_QK_TS = (1, 64, 2048)


def tp_crossover(rows):
    """From [T, H, one-shot us, two-shot us, NCCL us] rows: the first T where
    two-shot beats one-shot, and the first where the better fused form loses
    to NCCL all-reduce + norm (None when it never happens)."""
    two_wins = next((r[0] for r in rows if r[2] is not None and r[3] is not None and r[3] < r[2]), None)
    nccl_wins = next((r[0] for r in rows
                      if r[4] is not None and min(x for x in (r[2], r[3]) if x is not None) > r[4]), None)
    return {"twoshot_beats_oneshot_from_T": two_wins, "nccl_beats_fused_from_T": nccl_wins}


def tp_arm(ar, device, stream, world, rank, iters=100):
    """Per shape: the fused one-shot and two-shot pull kernels, and the
    unfused baseline (copy of the partial, NCCL all_reduce, then this
    library's add + RMSNorm with W = 1), each timed over `iters` calls with
    CUDA events on the launching stream, max over ranks.  Every rank takes the
    same steps in the same order."""
    import torch
    import torch.distributed as dist
    from tensor_allreduce_residual_ar_b200 import comm as C
    comm = C.Comm(8192 * 8192, device=device)
    oneshot_max = comm.tune_oneshot_max()          # the measured crossover, set on the communicator
    rows, worst = [], 0.0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(10):
            fn()
        torch.cuda.synchronize()
        barrier(device)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(iters):
                fn()
            ev1.record(stream)
        ev1.synchronize()
        return max_over_ranks(ev0.elapsed_time(ev1) / iters * 1e3, device)

    try:
        for T, H in TP_SHAPES:
            g = torch.Generator(device=device).manual_seed(7000 + T)          # same on every rank
            res = torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)
            w = (1 + 0.1 * torch.randn(H, generator=g, device=device)).to(torch.bfloat16)
            gp = torch.Generator(device=device).manual_seed(8000 + 131 * rank + T)
            part = (0.5 * torch.randn(T, H, generator=gp, device=device)).to(torch.bfloat16)
            out, rout = torch.empty_like(part), torch.empty_like(part)
            buf, ref, rref = torch.empty_like(part), torch.empty_like(part), torch.empty_like(part)

            def baseline():
                with torch.cuda.stream(stream):
                    buf.copy_(part)
                    dist.all_reduce(buf)
                    ar.ar_add_rmsnorm([buf], res, w, ref, rref, eps=1e-6)

            def fused(algo):
                return lambda: comm.allreduce_add_rmsnorm(part, res, w, out, rout, eps=1e-6, algo=algo,
                                                          stream=stream)
            us = {"nccl": timed(baseline)}
            for algo in ("oneshot", "twoshot"):
                if algo == "oneshot" and T * H * 2 > (8 << 20):
                    us[algo] = None
                    continue
                us[algo] = timed(fused(algo))
                torch.cuda.synchronize()
                d = ((out.float() - ref.float()).abs() / ref.float().abs().clamp_min(1e-2)).max().item()
                worst = max(worst, d)
            rows.append([T, H, None if us["oneshot"] is None else round(us["oneshot"], 2),
                         round(us["twoshot"], 2), round(us["nccl"], 2)])
            del part, res, w, out, rout, buf, ref, rref
        qk = []
        q_size, kv_size = 6144, 1024
        qs, ks = q_size // world, kv_size // world
        for T in TP_QK_TS:
            g = torch.Generator(device=device).manual_seed(9000 + T)
            qw = (1 + 0.1 * torch.randn(q_size, generator=g, device=device)).to(torch.bfloat16)
            kw = (1 + 0.1 * torch.randn(kv_size, generator=g, device=device)).to(torch.bfloat16)
            gp = torch.Generator(device=device).manual_seed(9500 + 131 * rank + T)
            qkv = torch.randn(T, qs + 2 * ks, generator=gp, device=device).to(torch.bfloat16)
            qo, ko = torch.empty((T, qs), dtype=torch.bfloat16, device=device), \
                torch.empty((T, ks), dtype=torch.bfloat16, device=device)

            def qk_baseline():
                # the unfused form: sums of squares, NCCL all_reduce, normalise
                with torch.cuda.stream(stream):
                    x = qkv.float()
                    ss = torch.stack([x[:, :qs].pow(2).sum(-1), x[:, qs:qs + ks].pow(2).sum(-1)], -1)
                    dist.all_reduce(ss)
                    qo.copy_(x[:, :qs] * torch.rsqrt(ss[:, :1] / q_size + 1e-6) * qw[rank * qs:(rank + 1) * qs])
                    ko.copy_(x[:, qs:qs + ks] * torch.rsqrt(ss[:, 1:] / kv_size + 1e-6) *
                             kw[rank * ks:(rank + 1) * ks])
            t_base = timed(qk_baseline)
            t_fused = timed(lambda: comm.qk_norm_sharded(qkv, qw, kw, qo, ko, q_size, kv_size, eps=1e-6,
                                                         stream=stream))
            qk.append([T, round(t_fused, 2), round(t_base, 2)])
        status = comm.status()
        # every rank's last exchange kernel has finished reading the others'
        # regions before any rank frees its own
        torch.cuda.synchronize()
        barrier(device)
    finally:
        comm.close()
    return {"norm_us": rows, "norm_fields": "T, H, one-shot, two-shot, copy + NCCL all_reduce + W=1 "
                                            "norm (us per call, max over ranks; bf16, one partial per rank)",
            **tp_crossover(rows), "max_rel_vs_nccl_path": round(worst, 5),
            "qk_us": qk, "qk_fields": "T, fused, torch sums + NCCL all_reduce + normalise",
            "oneshot_max_bytes": oneshot_max, "crossover_us": comm.crossover_us,
            "status": status}


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------

def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores (threads over
    row blocks), on the same workload, metric and unit; each step a bounded
    sample of the workload (every call, the first rows of each) so K + W
    steps take about two minutes."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    calls = workload_calls(args.workload)
    cpu = host_cpu()
    threads = cpu["nproc"]
    t_full, _, _ = oracle_sample(calls, 0.0, max_steps=1, threads=threads)   # one full step, timed
    total_budget = 120.0
    frac = min(1.0, total_budget / max(1e-9, t_full * (args.steps + args.warmup)))
    oracle_sample(calls, 0.0, max_steps=args.warmup, row_fraction=frac, threads=threads)
    el, n, step_bytes = oracle_sample(calls, float("inf"), max_steps=args.steps, row_fraction=frac,
                                      threads=threads)
    value = step_bytes * n / el / 1e9
    rows = "every row of each call" if frac >= 1.0 else f"the first {frac * 100:.3g}% of each call's rows"
    sample = (f"{n} steps of the {args.workload} workload ({len(calls)} call(s) each, {rows}), "
              f"C fp64 on {threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
            "n_gpus": world, "steps": n, "warmup": args.warmup, "ms_per_step": round(el / n * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": describe(args.workload)},
            "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": sample,
                             "value": round(value, 5), "unit": "GB/s", **cpu},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_exchange_launches(args):
    """Profiling mode for the multi-GPU kernels: the world-size-1 rank-form
    call (decode shape H = 8192, bf16, residual and residual_out) in the
    --exchange form, `--launches` times per --only-T token count (default 1),
    plain stream launches."""
    import torch
    import tensor_allreduce_residual_ar_b200 as ar
    from tensor_allreduce_residual_ar_b200 import comm as C
    device = torch.device("cuda", dist_env()[2])
    torch.cuda.set_device(device)
    ar.load_library()
    H = 8192
    Ts = args.only_T or [1]
    comm = C.Comm(max(Ts) * H, device=device)
    try:
        g = torch.Generator(device=device).manual_seed(4243)
        w = (torch.randn(H, generator=g, device=device) * 0.1).to(torch.bfloat16)
        for T in Ts:
            p_, r_ = [torch.randn(T, H, generator=g, device=device).to(torch.bfloat16) for _ in range(2)]
            y, ro = torch.empty_like(p_), torch.empty_like(p_)
            for _ in range(args.launches):
                comm.allreduce_add_rmsnorm(p_, r_, w, y, ro, eps=1e-6, gemma=True, algo=args.exchange)
        torch.cuda.synchronize()
        if comm.status() != 0:
            raise RuntimeError("an exchange wait timed out")
    finally:
        comm.close()
    print(json.dumps({"launches": args.launches * len(Ts), "exchange": args.exchange, "T": Ts, "H": H}))
    return 0


def run_launches(args):
    """Profiling mode: every call of the workload `--launches` times, plain
    stream launches (no graph, no timing), for a profiler to capture."""
    import torch
    import tensor_allreduce_residual_ar_b200 as ar
    if args.exchange:
        return run_exchange_launches(args)
    device = torch.device("cuda", dist_env()[2])
    torch.cuda.set_device(device)
    ar.load_library()
    calls = workload_calls(args.workload)
    if args.only_T:
        calls = [c for c in calls if c[2] in args.only_T]
    if args.force_plan:
        variant = 2 if args.workload == "qk" else 1 if args.workload == "fp8" else 0
        if ar.ar_plan_force(variant, args.force_plan) != 0:
            raise ValueError(f"plan {args.force_plan} is not a plan of the {args.workload} workload")
    bufs = [CallBuffers(c, device) for c in calls]
    for _ in range(args.launches):
        for b in bufs:
            b.run(ar)
    torch.cuda.synchronize()
    print(json.dumps({"launches": args.launches * len(bufs), "workload": args.workload,
                      "calls": [[c[2], c[3], plan_of(ar, c)] for c in calls]}))
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    import tensor_allreduce_residual_ar_b200 as ar

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    ar.load_library()
    stream = torch.cuda.Stream(device)

    calls = workload_calls(args.workload)
    step_bytes = sum(call_bytes(c) for c in calls)
    R = rotation_sets(step_bytes)
    base = [CallBuffers(c, device, seed_offset=rank) for c in calls]
    sets = [base] + [[CallBuffers(c, device, inputs=b.inp) for c, b in zip(calls, base)]
                     for _ in range(R - 1)]
    with torch.cuda.stream(stream):
        for s in sets:
            for b in s:
                b.run(ar)   # first calls outside capture (device attributes)
    torch.cuda.synchronize()
    graphs = capture_step_graphs(ar, sets, stream)

    # warm-up: W steps, then enough untimed steps to bring clocks to load
    time_graphs(graphs, max(3, args.warmup), stream)
    est = time_graphs(graphs, 20, stream) / 20
    spin = int(min(20000, max(10, args.spin_seconds / max(est, 1e-7))))   # load before timing
    sampler = ClockSampler(device.index)
    with sampler:
        time_graphs(graphs, spin, stream)
        barrier(device)
        torch.cuda.synchronize()
        el = time_graphs(graphs, args.steps, stream, label="bench_timed")
        torch.cuda.synchronize()
        barrier(device)
    el_max = max_over_ranks(el, device)
    value = weak_scaling_value(step_bytes, world, args.steps, el_max)
    peak, peak_src = load_peaks()
    per_rank_gbs = step_bytes * args.steps / el_max / 1e9
    launches = args.steps * len(calls)

    # end-to-end through the public call with host buffers
    e2e_steps = max(3, min(args.steps, 50))
    e_el, h2d, d2h = e2e_measure(ar, device, stream, calls, e2e_steps)
    e_el = max_over_ranks(e_el, device)
    e2e_value = weak_scaling_value(step_bytes, world, e2e_steps, e_el)

    line = {"metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el_max / args.steps * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded torch.randn, the workload's distributions)",
            "config": {"workload": describe(args.workload), "calls_per_step": len(calls),
                       "bytes_per_step": step_bytes, "storage": ",".join(sorted({c[3] for c in calls})),
                       "plans": sorted({plan_of(ar, c) for c in calls}),
                       "l2": (f"{R} rotating buffer sets, each reused after "
                              f">{(R - 1) * step_bytes / 2**20:.0f} MiB of other traffic"
                              if R > 1 else "inputs larger than L2 (126 MiB)"),
                       "parallelism": f"replicas x{world}, no collective"},
            "us_per_call": round(el_max / args.steps / len(calls) * 1e6, 3),
            "gpu_launches": launches,
            "roofline": {"bound": "hbm", "achieved": round(per_rank_gbs, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(per_rank_gbs / peak, 4),
                         "peak_source": "measured hbm_gbs" if peak_src == "measured"
                         else "fallback 6.65 TB/s",
                         "frac_of_8TBps": round(per_rank_gbs / NOMINAL_HBM_GBS, 4),
                         "traffic": ncu_traffic(args.workload),
                         "kernel": "norm_rows_kernel" if args.workload != "qk" else "qk_norm_kernel"},
            "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "clocks": sampler.summary()}

    del graphs
    if world > 1 and not args.no_tp:
        # the multi-GPU form itself: fused exchange kernels against NCCL
        try:
            line["tp"] = tp_arm(ar, device, stream, world, rank)
        except Exception as e:            # reported, never hidden
            line["tp"] = {"error": f"{type(e).__name__}: {str(e)[:300]}"}
    # Every collective is done: the ranks part here, so that rank 0's
    # sweep and oracle timing below (no collectives, a minute or more) keep
    # no other rank waiting in a barrier against the group's timeout.
    if world > 1:
        barrier(device)
        dist.destroy_process_group()
    if rank != 0:
        return 0
    if not args.no_sweep:
        sweep = run_sweep(ar, device, stream, args, peak_src)
        line["sweep_summary"] = sweep_summary(sweep, peak_src)
    if world == 1 and not args.no_cpu_baseline:
        cpu = host_cpu()
        threads = cpu["nproc"]
        el_c, n_c, sb = oracle_sample(calls, args.cpu_seconds, threads=threads)
        el_1, n_1, sb_1 = oracle_sample(calls, 0.0, max_steps=1, threads=1,
                                        row_fraction=min(1.0, 1.0 / max(1, threads)))
        line["cpu_baseline"] = {
            "value": round(sb * n_c / el_c / 1e9, 5), "unit": "GB/s", "cores": threads,
            "kind": "oracle", **cpu,
            "value_1_thread": round(sb_1 * n_1 / el_1 / 1e9, 5),
            "sample": f"{n_c} full steps of the {args.workload} workload in {el_c:.1f} s, C fp64 "
                      f"on {threads} threads over row blocks; value_1_thread: one step on the "
                      f"first 1/{max(1, threads)} of the rows, one thread"}
    print(json.dumps(line), flush=True)
    return 0


def sweep_names(args):
    return ["tiny", "decode", "qk", "fp8", "prefill"] if args.sweep == "all" else \
        [n for n in args.sweep.split(",") if n]


def exchange_sweep(ar, device, stream, Ts=None, reps=20):
    """The exchange kernels' own cost on one GPU: the rank-form communicator
    at world size 1 runs the multi-GPU kernels (the partial staged into the
    communicator's region, the sys-scope flag barrier, then the fused add +
    norm reading the staged rows), with no NVLink in the path.  Per token
    count of the decode shape (H = 8192, bf16, residual and residual_out),
    and the prefill-sized T = 8192 at H = 4096: device time per call of the
    plain fused call with one partial, of the one-shot and of the two-shot
    form, each in a CUDA graph over rotating buffer sets as in the sweep."""
    import torch
    from tensor_allreduce_residual_ar_b200 import comm as C
    shapes = [(T, 8192) for T in (Ts or (1, 16, 80, 512))] + ([] if Ts else [(8192, 4096)])
    rows = []
    for T, H in shapes:
        nbytes = T * H * 2 * 4 + H * 2          # partial, residual, y, residual_out
        R = min(rotation_sets(nbytes), 2048)
        g = torch.Generator(device=device).manual_seed(4242 + T)
        w = (torch.randn(H, generator=g, device=device) * 0.1).to(torch.bfloat16)
        sets = []
        for _ in range(R):
            t = [(torch.randn(T, H, generator=g, device=device)).to(torch.bfloat16) for _ in range(2)]
            sets.append((t[0], t[1], torch.empty_like(t[0]), torch.empty_like(t[0])))
        comm = C.Comm(T * H, device=device)
        res = {"T": T, "H": H, "sets": R}
        try:
            forms = {
                "plain": lambda b: ar.ar_add_rmsnorm([b[0]], b[1], w, b[2], b[3], eps=1e-6, gemma=True,
                                                     stream=stream),
                "oneshot": lambda b: comm.allreduce_add_rmsnorm(b[0], b[1], w, b[2], b[3], eps=1e-6,
                                                                gemma=True, algo="oneshot", stream=stream),
                "twoshot": lambda b: comm.allreduce_add_rmsnorm(b[0], b[1], w, b[2], b[3], eps=1e-6,
                                                                gemma=True, algo="twoshot", stream=stream),
            }
            for name, f in forms.items():
                with torch.cuda.stream(stream):
                    f(sets[0])
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    with torch.cuda.graph(graph, stream=stream):
                        for b in sets:
                            f(b)
                time_graphs([graph], 2, stream)
                sec = time_graphs([graph], reps, stream) / (reps * R)
                res[name + "_us"] = round(sec * 1e6, 3)
                del graph
            torch.cuda.synchronize()
            if comm.status() != 0:
                raise RuntimeError("an exchange wait timed out")
        finally:
            comm.close()
        rows.append(res)
        del sets
        torch.cuda.empty_cache()
    # the sharded QK-norm's exchange (only each token's two sums of squares
    # cross ranks) at world size 1, against the plain call with one shard
    for T in (Ts or (1, 64, 2048)):
        q_size, kv_size = 6144, 1024
        row = q_size + 2 * kv_size
        nbytes = T * (q_size + kv_size) * 2 * 2
        R = min(rotation_sets(nbytes), 2048)
        g = torch.Generator(device=device).manual_seed(4343 + T)
        qw = (1 + 0.1 * torch.randn(q_size, generator=g, device=device)).to(torch.bfloat16)
        kw = (1 + 0.1 * torch.randn(kv_size, generator=g, device=device)).to(torch.bfloat16)
        sets = []
        for _ in range(R):
            x = torch.randn(T, row, generator=g, device=device).to(torch.bfloat16)
            sets.append((x, torch.empty(T, q_size, dtype=torch.bfloat16, device=device),
                         torch.empty(T, kv_size, dtype=torch.bfloat16, device=device)))
        comm = C.Comm(T * row, device=device)
        res = {"T": T, "H": q_size + kv_size, "sets": R, "qk": True}
        try:
            forms = {
                "plain": lambda b: ar.qk_norm_sharded([b[0]], qw, kw, [b[1]], [b[2]], q_size, kv_size,
                                                      eps=1e-6, stream=stream),
                "exchange": lambda b: comm.qk_norm_sharded(b[0], qw, kw, b[1], b[2], q_size, kv_size,
                                                           eps=1e-6, stream=stream),
            }
            for name, f in forms.items():
                with torch.cuda.stream(stream):
                    f(sets[0])
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    with torch.cuda.graph(graph, stream=stream):
                        for b in sets:
                            f(b)
                time_graphs([graph], 2, stream)
                sec = time_graphs([graph], reps, stream) / (reps * R)
                res[name + "_us"] = round(sec * 1e6, 3)
                del graph
            torch.cuda.synchronize()
            if comm.status() != 0:
                raise RuntimeError("an exchange wait timed out")
        finally:
            comm.close()
        rows.append(res)
        del sets
        torch.cuda.empty_cache()
    return rows


def run_sweep(ar, device, stream, args, peak_src):
    """The per-call sweep, printed as text lines (and written as JSON with
    --sweep-out)."""
    names = sweep_names(args)
    sweep = per_call_sweep(ar, device, stream, [n for n in names if n != "exchange"], Ts=args.sweep_T)
    if "exchange" in names:
        sweep["exchange"] = exchange_sweep(ar, device, stream, Ts=args.sweep_T)
        for r in sweep["exchange"]:
            if r.get("qk"):
                print(f"sweep exchange qk T={r['T']} q+kv={r['H']} bf16: plain {r['plain_us']} us, "
                      f"exchange {r['exchange_us']} us (world size 1)", flush=True)
                continue
            print(f"sweep exchange T={r['T']} H={r['H']} bf16: plain {r['plain_us']} us, one-shot "
                  f"{r['oneshot_us']} us, two-shot {r['twoshot_us']} us (world size 1)", flush=True)
    for name, rows in sweep.items():
        if name == "exchange":
            continue
        for r in rows:
            hot = f" (hot L2 {r['us_hot_l2']} us)" if "us_hot_l2" in r else ""
            print(f"sweep {name} T={r['T']} {r['dtype']}: {r['us']} us{hot}, {r['GBps']} GB/s, "
                  f"{r['frac_of_peak']} of the {peak_src} peak, {r['frac_of_8TBps']} of 8 TB/s, "
                  f"plan {r['plan']}", flush=True)
    if args.sweep_out:
        with open(args.sweep_out, "w") as f:
            json.dump(sweep, f, indent=1)
    return sweep


def run_sweep_only(args):
    """Sweep mode: only the per-call sweep of the --sweep workloads, at the
    --sweep-T token counts if given, with --force-plan applied to every call
    of the workloads' variant if given; one GPU, nothing else timed."""
    import torch
    import tensor_allreduce_residual_ar_b200 as ar
    device = torch.device("cuda", dist_env()[2])
    torch.cuda.set_device(device)
    ar.load_library()
    _, peak_src = load_peaks()
    if args.force_plan:
        for name in sweep_names(args):
            variant = 2 if name == "qk" else 1 if name == "fp8" else 0
            if ar.ar_plan_force(variant, args.force_plan) != 0:
                raise ValueError(f"plan {args.force_plan} is not a plan of the {name} workload")
    stream = torch.cuda.Stream(device)
    run_sweep(ar, device, stream, args, peak_src)
    return 0


def sweep_summary(sweep, peak_src="measured"):
    """The sweep rows the targets are about, compact: per-call us and the
    fractions of the copy peak (measured, or the fallback) and of 8 TB/s."""
    out = {}

    def pick(name, T, dtype="bf16"):
        for r in sweep.get(name, []):
            if r["T"] == T and r["dtype"] == dtype:
                return [r["us"], r["frac_of_peak"], r["frac_of_8TBps"], r["plan"]]
        return None

    for key, args in (("prefill_T8192", ("prefill", 8192)), ("fp8_T2048", ("fp8", 2048)),
                      ("fp8_T8192", ("fp8", 8192)), ("fp8_T32768", ("fp8", 32768)),
                      ("qk_T2048", ("qk", 2048)), ("tiny_T16", ("tiny", 16))):
        v = pick(*args)
        if v is not None:
            out[key] = v
    dec = sweep.get("decode", [])
    if dec:
        out["decode_us_min_max"] = [min(r["us"] for r in dec), max(r["us"] for r in dec)]
        out["decode_T80_bf16"] = pick("decode", 80)
    out["fields"] = f"us/call, frac of the {peak_src} copy peak, frac of 8 TB/s, plan"
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "decode", "tiny", "fp8", "qk"], default="prefill")
    ap.add_argument("--sweep", default="all", help="workloads for the per-call sweep (comma list or all)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--sweep-out", default=None, help="also write the full sweep as JSON here")
    ap.add_argument("--sweep-only", action="store_true",
                    help="run only the per-call sweep (with --sweep-T, --force-plan) and exit")
    ap.add_argument("--sweep-T", type=int, nargs="*", default=None,
                    help="token counts for the sweep instead of each workload's own")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tp", action="store_true", help="N > 1: skip the multi-GPU exchange arm")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--spin-seconds", type=float, default=0.5,
                    help="untimed load before the timed region (clocks settle, sampler runs)")
    ap.add_argument("--launches", type=int, default=0,
                    help="profiling mode: run every call this many times and exit")
    ap.add_argument("--exchange", choices=["oneshot", "twoshot"], default=None,
                    help="profiling mode: the multi-GPU kernel at world size 1 instead of a workload")
    ap.add_argument("--only-T", type=int, nargs="*", default=None,
                    help="profiling mode: restrict to these T")
    ap.add_argument("--force-plan", type=int, default=0,
                    help="profiling and sweep modes: run every call with this dispatch plan")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.launches:
        return run_launches(args)
    if args.sweep_only:
        return run_sweep_only(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
