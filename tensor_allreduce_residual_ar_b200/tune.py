"""Measure every dispatch plan on each shape and write the plan table.

    python -m tensor_allreduce_residual_ar_b200.tune [--out plan_table.json] [--reps 10]

For each shape of the five workloads (and any --extra shapes) every plan that
is valid for the variant is forced in turn, a CUDA graph holding the call
once per rotating buffer set (enough sets that a set is reused only after
more than twice the L2 size of other traffic, or inputs larger than L2) is
replayed, and the device time per call is taken with CUDA events.  The
fastest plan wins; consecutive measured T values become T ranges
(prev_T, T], the largest measured T extending to any larger T.  The table is
what ``ar_plan_load`` reads; a timing report goes next to it.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

from . import binding as ar
from . import workloads as wl

L2_BYTES = 126 * 1024 * 1024
NORM_PLANS = (1, 2, 3, 4, 5, 6, 7, 8, 9, 10)
QK_PLANS = (11, 12, 13, 14, 15, 16, 17, 18)
T_MAX = 1 << 40


class Slab:
    """One device allocation carved into 256-byte aligned views."""

    def __init__(self, nbytes: int, device):
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.off = 0

    def take(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nb = n * torch.empty((), dtype=dtype).element_size()
        v = self.buf[self.off:self.off + nb].view(dtype).view(*shape)
        self.off += (nb + 255) // 256 * 256
        return v


def _sets(step_bytes: int) -> int:
    if step_bytes >= 4 * L2_BYTES:
        return 1
    return min(4096, int(2 * L2_BYTES // step_bytes) + 2)


def _norm_sets(shape, device):
    variant, dtype, W, H, T, has_res, write_res = shape
    td = {"bf16": torch.bfloat16, "fp16": torch.float16}[dtype]
    base = wl.make_norm_inputs(wl.FP8 if variant == 1 else wl.DECODE, T, dtype, W=W, H=H,
                               residual=has_res, device=device)
    nbytes = wl.norm_bytes(T, H, W, has_res, write_res, fp8=variant == 1)
    R = _sets(nbytes)
    per = (W + 4) * (T * H * 2 + 256) + H * 2 + T * H + T * (H // 128) * 4 + 4096
    slab = Slab(per * R, device)
    sets = []
    for _ in range(R):
        parts = [slab.take((T, H), td) for _ in range(W)]
        for d, s in zip(parts, base.partials):
            d.copy_(s)
        res = slab.take((T, H), td) if has_res else None
        if res is not None:
            res.copy_(base.residual)
        w = slab.take((H,), td)
        w.copy_(base.weight)
        out = slab.take((T, H), td)
        rout = slab.take((T, H), td) if write_res else None
        if variant == 1:
            q = slab.take((T, H), torch.uint8)
            sc = slab.take((T, H // 128), torch.float32)
            sets.append(lambda parts=parts, res=res, w=w, q=q, sc=sc, out=out, rout=rout:
                        ar.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q, sc, out, rout, eps=1e-6))
        else:
            sets.append(lambda parts=parts, res=res, w=w, out=out, rout=rout:
                        ar.ar_add_rmsnorm(parts, res, w, out, rout, eps=1e-6, gemma=True))
    return sets, nbytes, slab


def _qk_sets(shape, device):
    _, dtype, W, qkv_size, T, q_size, kv_size = shape
    td = {"bf16": torch.bfloat16, "fp16": torch.float16}[dtype]
    base = wl.make_qk_inputs(wl.QK, T, dtype, W=W, q_size=q_size, kv_size=kv_size, device=device)
    nbytes = wl.qk_bytes(T, W, q_size, kv_size)
    R = _sets(nbytes)
    qs, ks = q_size // W, kv_size // W
    per = W * ((T * (qs + 2 * ks) * 2 + 256) + (T * qs * 2 + 256) + (T * ks * 2 + 256)) + \
        (q_size + kv_size) * 2 + 1024
    slab = Slab(per * R, device)
    sets = []
    for _ in range(R):
        qkv = [slab.take((T, qs + 2 * ks), td) for _ in range(W)]
        for d, s in zip(qkv, base.qkv):
            d.copy_(s)
        qw, kw = slab.take((q_size,), td), slab.take((kv_size,), td)
        qw.copy_(base.q_weight)
        kw.copy_(base.k_weight)
        qo = [slab.take((T, qs), td) for _ in range(W)]
        ko = [slab.take((T, ks), td) for _ in range(W)]
        sets.append(lambda qkv=qkv, qw=qw, kw=kw, qo=qo, ko=ko:
                    ar.qk_norm_sharded(qkv, qw, kw, qo, ko, q_size, kv_size, eps=1e-6))
    return sets, nbytes, slab


def time_plan(variant: int, plan: int, sets, reps: int, stream) -> float:
    """Seconds per call with `plan` forced."""
    assert ar.ar_plan_force(variant, plan) == 0
    try:
        with torch.cuda.stream(stream):
            for f in sets:
                f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in sets:
                f()
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
        b.synchronize()
        del g
        return a.elapsed_time(b) / 1e3 / (reps * len(sets))
    finally:
        ar.ar_plan_force(variant, 0)


# Token counts measured beyond the workloads' own, so that calls of those
# shapes at other lengths get a measured plan rather than the neighbouring
# one's (the prefill shape at decode and long-prefill lengths; QK past 2048
# tokens, where the register load-ahead plan overtakes the shared-memory ring).
PREFILL_EXTRA_TS = (16, 256, 2048, 32768)
QK_EXTRA_TS = (4096, 8192, 32768)


def default_shapes():
    out = []
    for dt in wl.DECODE.dtypes:
        for T in wl.DECODE.Ts:
            out.append((0, dt, 4, 8192, T, True, True))
    out.append((0, "bf16", 2, 4096, 16, True, True))
    for T in sorted(set(wl.PREFILL.Ts) | set(PREFILL_EXTRA_TS)):
        out.append((0, "bf16", 8, 4096, T, True, False))
    for T in wl.FP8.Ts:
        out.append((1, "bf16", 4, 5120, T, True, True))
    for T in sorted(set(wl.QK.Ts) | set(QK_EXTRA_TS)):
        out.append((2, "bf16", 8, 6144 + 1024, T, 6144, 1024))
    return out


def tune(shapes, reps: int, device) -> tuple[dict, list]:
    ar.load_library()
    ar.ar_plan_load(None)     # measure without any table
    stream = torch.cuda.Stream(device)
    report = []
    best = {}
    for shape in shapes:
        variant, dtype, W, H, T = shape[:5]
        if variant == 2:
            sets, nbytes, slab = _qk_sets(shape, device)
            plans = QK_PLANS
        else:
            sets, nbytes, slab = _norm_sets(shape, device)
            plans = NORM_PLANS
        times = {}
        for pl in plans:
            times[pl] = time_plan(variant, pl, sets, reps, stream)
        win = min(times, key=times.get)
        best[(variant, wl.DTYPE_CODE[dtype], W, H, T)] = win
        report.append({"variant": variant, "dtype": dtype, "W": W, "H": H, "T": T, "bytes": nbytes,
                       "sets": len(sets), "us": {str(k): round(v * 1e6, 3) for k, v in times.items()},
                       "best": win, "best_GBps": round(nbytes / times[win] / 1e9, 1)})
        print(json.dumps(report[-1]), flush=True)
        del sets, slab
        torch.cuda.empty_cache()
    return table_from_best(best), report


def table_from_best(best: dict) -> dict:
    """{(variant, dtype, W, H, T): plan} -> plan-table entries: for each key,
    consecutive measured T become ranges (prev_T, T] (the first from 0, the
    last open-ended); neighbouring ranges with the same plan are merged."""
    entries = []
    for key in sorted({k[:4] for k in best}):
        Ts = sorted(k[4] for k in best if k[:4] == key)
        prev = None
        for i, T in enumerate(Ts):
            lo = 0 if prev is None else prev + 1
            hi = T if i + 1 < len(Ts) else T_MAX
            plan = best[key + (T,)]
            e = entries[-1] if entries else None
            if e and (e["variant"], e["dtype"], e["W"], e["H"]) == key and e["plan"] == plan:
                e["t_hi"] = hi
            else:
                entries.append({"variant": key[0], "dtype": key[1], "W": key[2], "H": key[3],
                                "t_lo": lo, "t_hi": hi, "plan": plan})
            prev = T
    return {"entries": entries}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--out", default=os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                  "plan_table.json"))
    ap.add_argument("--report", default=os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                     "plan_report.jsonl"),
                    help="per-plan microseconds of every tuned shape (one JSON line per shape)")
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args(argv)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    table, report = tune(default_shapes(), a.reps, device)
    with open(a.out, "w") as f:
        json.dump(table, f, indent=1)
        f.write("\n")
    if a.report:
        with open(a.report, "w") as f:
            for r in report:
                f.write(json.dumps(r) + "\n")
    print(f"wrote {len(table['entries'])} entries to {a.out}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
