"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on
the same seeded inputs, at the five workloads' sizes (full comparison where
the oracle takes seconds, sampled rows beyond that), with every dispatch
plan forced on ragged shapes, and on the edge cases the method has (no
residual, dead residual, in-place residual, W = 1 and 16, the smallest and
largest H, cancellation, fp16 subnormal outputs, all-zero FP8 groups).
Every output buffer carries a guard band that must come back untouched."""
import numpy as np
import pytest
import torch

import parity as P
from tensor_allreduce_residual_ar_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD = 512
SENT16 = 0x5A5A
NORM_PLANS = (1, 2, 3, 4, 5, 6, 7, 8, 9, 10)
QK_PLANS = (11, 12, 13, 14, 15, 16, 17, 18)
TD = {"bf16": torch.bfloat16, "fp16": torch.float16}


class Guarded:
    """A device buffer of n elements followed by a guard band, pre-filled
    with a sentinel so unwritten elements and overruns both show."""

    def __init__(self, shape, dtype, sentinel):
        n = int(np.prod(shape))
        raw_dtype = {torch.bfloat16: torch.int16, torch.float16: torch.int16}.get(dtype, dtype)
        self.buf = torch.full((n + GUARD,), sentinel, dtype=raw_dtype, device="cuda")
        self.n = n
        self.sentinel = sentinel
        self.view = self.buf[:n].view(dtype).view(*shape) if raw_dtype != dtype else self.buf[:n].view(*shape)

    def guard_ok(self):
        g = self.buf[self.n:]
        return bool((g == self.sentinel).all().item())


@pytest.fixture(autouse=True)
def _reset_plans(lib):
    yield
    for v in range(3):
        lib.ar_plan_force(v, 0)


def run_norm(lib, inp, *, write_res=None, inplace=False, plan=None, residual=True):
    dev = "cuda"
    td = TD[inp.dtype]
    parts = [p.to(dev) for p in inp.partials]
    res = inp.residual.to(dev) if (inp.residual is not None and residual) else None
    w = inp.weight.to(dev)
    write_res = inp.write_residual if write_res is None else write_res
    out = Guarded((inp.T, inp.H), td, SENT16)
    rout = None
    if write_res and not inplace:
        rout = Guarded((inp.T, inp.H), td, SENT16)
    if plan is not None:
        assert lib.ar_plan_force(0, plan) == 0
    res_before = res.clone() if res is not None else None
    lib.ar_add_rmsnorm(parts, res, w, out.view, res if inplace else (rout.view if rout else None),
                       eps=inp.eps, gemma=inp.gemma)
    torch.cuda.synchronize()
    assert out.guard_ok()
    got = {"y": P.to_bits(out.view)}
    if rout is not None:
        assert rout.guard_ok()
        got["r"] = P.to_bits(rout.view)
    if inplace:
        got["r"] = P.to_bits(res)
    elif res is not None:
        assert torch.equal(res, res_before), "residual input was modified"
    return got


def check_norm(lib, inp, **kw):
    got = run_norm(lib, inp, **kw)
    o = P.oracle_norm(inp) if kw.get("residual", True) else P.oracle_norm(
        wl.NormInputs(inp.partials, None, inp.weight, inp.T, inp.H, inp.W, inp.dtype, inp.eps,
                      inp.gemma, inp.write_residual))
    stats = P.check_y(got["y"], o["y"], inp.dtype)
    if "r" in got:
        P.check_res(got["r"], o["r"], inp.dtype)
    return stats


# ----------------------------------------------------------------------------
# the five workloads
# ----------------------------------------------------------------------------

def test_tiny(lib, parity_report):
    st = check_norm(lib, wl.make_norm_inputs(wl.TINY, 16))
    assert st["ulp_clause"] == 0
    parity_report("tiny T=16 y", st)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("T", wl.DECODE.Ts)
def test_decode_window(lib, T, dtype, parity_report):
    st = check_norm(lib, wl.make_norm_inputs(wl.DECODE, T, dtype))
    if dtype == "bf16":
        assert st["ulp_clause"] == 0
    parity_report(f"decode T={T} {dtype} y", st)


def test_prefill_dead_residual_full(lib, parity_report):
    inp = wl.make_norm_inputs(wl.PREFILL, 8192)
    assert not inp.write_residual
    st = check_norm(lib, inp)
    assert st["ulp_clause"] == 0
    parity_report("prefill T=8192 y", st)


def run_fp8(lib, inp, *, with_y=True, with_res=True, plan=None):
    """One FP8-variant call on guarded buffers.  With inp.residual None it is
    the no-residual form (r is the plain sum of the partials); residual_out
    is still written when with_res is set."""
    dev = "cuda"
    T, H = inp.T, inp.H
    parts = [p.to(dev) for p in inp.partials]
    res = inp.residual.to(dev) if inp.residual is not None else None
    w = inp.weight.to(dev)
    q = Guarded((T, H), torch.uint8, 0xA5)
    s = Guarded((T, H // 128), torch.float32, -7.0)
    y = Guarded((T, H), TD[inp.dtype], SENT16) if with_y else None
    r = Guarded((T, H), TD[inp.dtype], SENT16) if with_res else None
    if plan is not None:
        assert lib.ar_plan_force(1, plan) == 0
    lib.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q.view, s.view, y.view if y else None,
                                       r.view if r else None, eps=inp.eps, gemma=inp.gemma)
    torch.cuda.synchronize()
    for b in (q, s, y, r):
        if b is not None:
            assert b.guard_ok()
    return (q.view.cpu().numpy(), s.view.cpu().numpy(),
            P.to_bits(y.view) if y else None, P.to_bits(r.view) if r else None)


def check_fp8(lib, inp, rows=None, **kw):
    q, s, y, r = run_fp8(lib, inp, **kw)
    o = P.oracle_norm(inp, rows=rows)
    if rows is not None:
        q, s = q[rows], s[rows]
        y = y[rows] if y is not None else None
        r = r[rows] if r is not None else None
    st = P.check_fp8(q, s, o["y"])
    if y is not None:
        sy = P.check_y(y, o["y"], inp.dtype)
        if inp.dtype == "bf16":
            assert sy["ulp_clause"] == 0
        st.update({"y_" + k: v for k, v in sy.items()})
    if r is not None:
        P.check_res(r, o["r"], inp.dtype)
    return st


@pytest.mark.parametrize("T", wl.FP8.Ts)
def test_fp8_group_sweep(lib, T, parity_report):
    inp = wl.make_norm_inputs(wl.FP8, T)
    rows = None
    if T > 2048:   # sampled rows at the largest sizes: first, last and 62 spread
        rng = np.random.default_rng(T)
        rows = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 62, replace=False)]))
    st = check_fp8(lib, inp, rows=rows)
    parity_report(f"fp8 T={T} codes/scales", st)


@pytest.mark.parametrize("plan", NORM_PLANS)
def test_fp8_no_residual_every_plan(lib, plan):
    """The no-residual FP8 site (all_reduce -> rms_norm -> per-group quant):
    residual NULL, so r is the plain sum of the partials.  Codes, scales,
    the 16-bit y and residual_out (the sum itself) against the oracle, on
    row, persistent and bulk-staged plans, ragged shapes included."""
    for T, H, W in ((1, 128, 1), (7, 640, 3), (67, 5120, 4), (300, 2048, 8)):
        inp = wl.make_norm_inputs(wl.FP8, T, W=W, H=H, residual=False, seed=3000 + T + H + W)
        assert inp.residual is None
        st = check_fp8(lib, inp, plan=plan)
        assert st["scale_max_rel"] <= P.SCALE_RTOL


@pytest.mark.parametrize("T", wl.QK.Ts)
def test_qk_sharded(lib, T, parity_report):
    st = check_qk(lib, wl.make_qk_inputs(wl.QK, T))
    assert st["ulp_clause"] == 0
    parity_report(f"qk T={T} q,k", st)


def run_qk(lib, inp, plan=None):
    dev = "cuda"
    W, qs, ks = inp.W, inp.q_size // inp.W, inp.kv_size // inp.W
    qkv = [x.to(dev) for x in inp.qkv]
    before = [x.clone() for x in qkv]
    qo = [Guarded((inp.T, qs), TD[inp.dtype], SENT16) for _ in range(W)]
    ko = [Guarded((inp.T, ks), TD[inp.dtype], SENT16) for _ in range(W)]
    if plan is not None:
        assert lib.ar_plan_force(2, plan) == 0
    lib.qk_norm_sharded(qkv, inp.q_weight.to(dev), inp.k_weight.to(dev), [b.view for b in qo],
                        [b.view for b in ko], inp.q_size, inp.kv_size, eps=inp.eps)
    torch.cuda.synchronize()
    for b in qo + ko:
        assert b.guard_ok()
    for a, b in zip(qkv, before):
        assert torch.equal(a, b), "qkv (including v) must not be modified"
    return [P.to_bits(b.view) for b in qo], [P.to_bits(b.view) for b in ko]


def check_qk(lib, inp, plan=None):
    """Every shard's q and k outputs against the oracle; returns the worst
    statistics over all of them."""
    qo, ko = run_qk(lib, inp, plan)
    q64, k64 = P.oracle_qk(inp)
    worst = {"max_rel": 0.0, "p9999_rel": 0.0, "ulp_clause": 0}
    for w in range(inp.W):
        for st in (P.check_y(qo[w], q64[w], inp.dtype, f"q_out[{w}]"),
                   P.check_y(ko[w], k64[w], inp.dtype, f"k_out[{w}]")):
            worst["max_rel"] = max(worst["max_rel"], st["max_rel"])
            worst["p9999_rel"] = max(worst["p9999_rel"], st["p9999_rel"])
            worst["ulp_clause"] += st["ulp_clause"]
    return worst


# ----------------------------------------------------------------------------
# every plan, ragged shapes, edge cases
# ----------------------------------------------------------------------------

RAGGED = [(1, 8, 1), (3, 24, 3), (5, 1000, 5), (7, 4104, 16), (130, 2048, 2), (37, 8192, 4),
          (301, 5120, 8)]


@pytest.mark.parametrize("plan", NORM_PLANS)
@pytest.mark.parametrize("T,H,W", RAGGED)
def test_norm_every_plan_ragged(lib, plan, T, H, W):
    for dtype, gemma, res in (("bf16", False, True), ("fp16", True, False)):
        inp = wl.make_norm_inputs(wl.DECODE, T, dtype, W=W, H=H, seed=T * 131 + H + W)
        inp.gemma = gemma
        check_norm(lib, inp, plan=plan, residual=res)


def test_persistent_cluster_many_rows_per_cluster(lib):
    """Plan PERSIST_C2 on shapes where every 2-CTA cluster reduces about
    seven rows: the row partials' buffers and their barriers' phases are
    reused many times (fp32 partials for 16-bit outputs, fp64 for FP8)."""
    for dtype in ("bf16", "fp16"):
        inp = wl.make_norm_inputs(wl.DECODE, 1000, dtype, W=4, H=8192, seed=808)
        check_norm(lib, inp, plan=8)
    inp = wl.make_norm_inputs(wl.FP8, 1500, W=4, H=5120, seed=809)
    check_fp8(lib, inp, plan=8)


@pytest.mark.parametrize("plan", NORM_PLANS)
def test_norm_max_hidden(lib, plan):
    inp = wl.make_norm_inputs(wl.TINY, 3, W=2, H=65536, seed=65536)
    check_norm(lib, inp, plan=plan)


def test_inplace_residual(lib):
    inp = wl.make_norm_inputs(wl.DECODE, 33, "bf16", seed=5)
    check_norm(lib, inp, inplace=True)


def test_no_residual_and_dead_residual(lib):
    inp = wl.make_norm_inputs(wl.TINY, 9, seed=6)
    check_norm(lib, inp, residual=False, write_res=True)
    check_norm(lib, inp, write_res=False)


def test_permuted_partials_agree(lib):
    inp = wl.make_norm_inputs(wl.PREFILL, 64, seed=12)
    a = run_norm(lib, inp)
    perm = wl.NormInputs(inp.partials[::-1], inp.residual, inp.weight, inp.T, inp.H, inp.W,
                         inp.dtype, inp.eps, inp.gemma, inp.write_residual)
    b = run_norm(lib, perm)
    d = np.abs(P.ordinal16(a["y"]) - P.ordinal16(b["y"]))
    assert d.max() <= 1


def test_cancellation_is_exact(lib):
    """residual = 1024, P0 = tiny, P1 = -1024: r must equal P0 exactly (an
    fp32 running sum would lose P0 entirely)."""
    T, H = 4, 1024
    inp = wl.make_norm_inputs(wl.TINY, T, W=2, H=H, seed=77)
    res = inp.residual.clone()
    p0 = inp.partials[0].clone()
    p1 = inp.partials[1].clone()
    half = H // 2
    res[:, :half] = 1024.0
    p1[:, :half] = -1024.0
    p0[:, :half] = (torch.randn(T, half, generator=torch.Generator().manual_seed(1)) * 2.0 ** -20).to(
        torch.bfloat16)
    inp = wl.NormInputs([p0, p1], res, inp.weight, T, H, 2, "bf16", inp.eps, False, True)
    got = run_norm(lib, inp)
    assert np.array_equal(got["r"][:, :half], wl.bits(p0)[:, :half])
    o = P.oracle_norm(inp)
    P.check_y(got["y"], o["y"], "bf16")
    P.check_res(got["r"], o["r"], "bf16")


def test_fp16_subnormal_outputs(lib):
    inp = wl.make_norm_inputs(wl.DECODE, 6, "fp16", seed=31, H=2048)
    inp.weight = (torch.randn(2048, generator=torch.Generator().manual_seed(2)) * 1e-5).to(torch.float16)
    inp.gemma = False
    stats = check_norm(lib, inp)
    assert stats["ulp_clause"] > 0      # the subnormal range was really exercised


@pytest.mark.parametrize("plan", NORM_PLANS)
def test_fp8_every_plan_ragged(lib, plan):
    for T, H, W in ((1, 128, 1), (5, 640, 3), (67, 5120, 4), (300, 2048, 8)):
        inp = wl.make_norm_inputs(wl.FP8, T, W=W, H=H, seed=1000 + T + H)
        check_fp8(lib, inp, plan=plan)


@pytest.mark.parametrize("plan", NORM_PLANS)
def test_fp8_transposed_scales(lib, plan):
    """Scales written through strides: the transpose of a [H/128, T] buffer
    receives exactly the row-major scales, with the same codes and y; the
    buffer's guard bands stay intact."""
    T, H = 37, 5120
    G = H // 128
    inp = wl.make_norm_inputs(wl.FP8, T, W=4, H=H, seed=2024)
    q0, s0, y0, r0 = run_fp8(lib, inp, plan=plan)
    dev = "cuda"
    parts = [p.to(dev) for p in inp.partials]
    q = torch.empty((T, H), dtype=torch.uint8, device=dev)
    st = Guarded((G, T), torch.float32, -7.0)
    y = torch.empty((T, H), dtype=TD[inp.dtype], device=dev)
    assert lib.ar_plan_force(1, plan) == 0
    lib.ar_add_rmsnorm_quant_fp8_group(parts, inp.residual.to(dev), inp.weight.to(dev), q,
                                       st.view.t(), y, None, eps=inp.eps, gemma=inp.gemma)
    torch.cuda.synchronize()
    assert st.guard_ok()
    assert np.array_equal(st.view.t().cpu().numpy(), s0)
    assert np.array_equal(q.cpu().numpy(), q0)
    assert np.array_equal(P.to_bits(y), y0)


def test_fp8_zero_groups_and_options(lib):
    T, H = 6, 512
    inp = wl.make_norm_inputs(wl.FP8, T, W=2, H=H, seed=99)
    for t in (1, 4):
        inp.residual[t] = 0
        for p in inp.partials:
            p[t] = 0
    inp.residual[2, 128:256] = 0
    for p in inp.partials:
        p[2, 128:256] = 0
    q, s, _, _ = run_fp8(lib, inp, with_y=False, with_res=False)
    assert np.all(s[1] == 0) and np.all(q[1] == 0) and s[2, 1] == 0 and np.all(q[2, 128:256] == 0)
    check_fp8(lib, inp, with_y=False, with_res=False)
    inp.gemma = True
    check_fp8(lib, inp)


@pytest.mark.parametrize("plan", QK_PLANS)
def test_qk_every_plan(lib, plan):
    for T, W, q_size, kv_size in ((1, 8, 6144, 1024), (5, 8, 6144, 1024), (3, 1, 64, 32),
                                  (7, 2, 256, 128), (9, 16, 2048, 128), (33, 4, 512, 64),
                                  (600, 8, 6144, 1024)):   # several tokens per persistent CTA
        inp = wl.make_qk_inputs(wl.QK, T, W=W, q_size=q_size, kv_size=kv_size, seed=T + W + q_size)
        check_qk(lib, inp, plan=plan)


@pytest.mark.parametrize("plan", QK_PLANS)
def test_qk_in_place(lib, plan):
    """In-place form: q_out[w] / k_out[w] are the q / k column views of
    qkv[w]; those columns are overwritten with the normalised values and
    the v columns stay bit-identical."""
    for T, dtype in ((5, "bf16"), (300, "fp16")):
        inp = wl.make_qk_inputs(wl.QK, T, dtype, seed=500 + T)
        W, qs, ks = inp.W, inp.q_size // inp.W, inp.kv_size // inp.W
        qkv = [x.to("cuda").clone() for x in inp.qkv]
        v_before = [x[:, qs + ks:].clone() for x in qkv]
        assert lib.ar_plan_force(2, plan) == 0
        try:
            lib.qk_norm_sharded(qkv, inp.q_weight.to("cuda"), inp.k_weight.to("cuda"),
                                [x[:, :qs] for x in qkv], [x[:, qs:qs + ks] for x in qkv],
                                inp.q_size, inp.kv_size, eps=inp.eps)
            torch.cuda.synchronize()
        finally:
            lib.ar_plan_force(2, 0)
        q64, k64 = P.oracle_qk(inp)
        for w in range(W):
            P.check_y(P.to_bits(qkv[w][:, :qs].contiguous()), q64[w], dtype, f"q[{w}]")
            P.check_y(P.to_bits(qkv[w][:, qs:qs + ks].contiguous()), k64[w], dtype, f"k[{w}]")
            assert torch.equal(qkv[w][:, qs + ks:], v_before[w]), "v must not be modified"


def test_qk_rejects_strided_outputs(lib):
    inp = wl.make_qk_inputs(wl.QK, 4, seed=77)
    W, qs, ks = inp.W, inp.q_size // inp.W, inp.kv_size // inp.W
    qkv = [x.to("cuda") for x in inp.qkv]
    wide = torch.empty((4, 2 * qs), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        lib.qk_norm_sharded(qkv, inp.q_weight.to("cuda"), inp.k_weight.to("cuda"),
                            [wide[:, :qs]] * W, [torch.empty((4, ks), dtype=torch.bfloat16,
                                                              device="cuda")] * W,
                            inp.q_size, inp.kv_size, eps=inp.eps)


def test_qk_fp16(lib):
    inp = wl.make_qk_inputs(wl.QK, 17, "fp16", seed=3)
    check_qk(lib, inp)


def test_three_d_tokens_flatten(lib):
    """A [B, S, H] activation is T = B*S tokens (numel / H)."""
    inp = wl.make_norm_inputs(wl.TINY, 12, seed=8, H=1024)
    dev = "cuda"
    parts = [p.to(dev).view(3, 4, 1024) for p in inp.partials]
    res = inp.residual.to(dev).view(3, 4, 1024)
    out = torch.empty_like(res)
    rout = torch.empty_like(res)
    lib.ar_add_rmsnorm(parts, res, inp.weight.to(dev), out, rout, eps=inp.eps)
    torch.cuda.synchronize()
    o = P.oracle_norm(inp)
    P.check_y(P.to_bits(out.view(12, 1024)), o["y"], "bf16")
    P.check_res(P.to_bits(rout.view(12, 1024)), o["r"], "bf16")


def test_bulk_plan_wait_timeout_is_reported(lib):
    """A bulk-staged launch whose row never lands: its consumers' bounded
    wait runs out, the device status says AR_ETIMEDOUT, the context stays
    usable, and the next call is correct with a clean status."""
    inp = wl.make_norm_inputs(wl.PREFILL, 64, seed=41)
    assert lib.ar_device_status(True) == 0
    assert lib.ar_test_withhold_row(5) == 0
    run_norm(lib, inp, plan=6)                 # finishes after the 1 s limit
    assert lib.ar_device_status(True) == 5     # AR_ETIMEDOUT, now cleared
    assert lib.ar_device_status(True) == 0
    check_norm(lib, inp, plan=6)
    assert lib.ar_device_status(True) == 0


def test_bulk_plan_falls_back_when_rows_do_not_fit(lib):
    """W=16, H=8192: 17 rows of 16 KiB per stage do not fit twice in shared
    memory, so the bulk plan runs the persistent kernel instead."""
    inp = wl.make_norm_inputs(wl.DECODE, 9, "bf16", W=16, H=8192, seed=42)
    check_norm(lib, inp, plan=6)


@pytest.mark.parametrize("plan", (1, 5, 6))
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_cancellation_sweep_around_certificate(lib, plan, dtype):
    """residual = -(sum of partials) + delta * noise, rounded: r is small
    against the terms at every scale delta, so elements land on both sides
    of the fast-sum acceptance test and many take the exact fallback."""
    T, H, W = 16, 2048, 6
    gen = torch.Generator().manual_seed(7000 + plan)
    td = TD[dtype]
    parts = [torch.randn(T, H, generator=gen).to(td) for _ in range(W)]
    total = sum(p.double() for p in parts)
    scales = torch.tensor([1e-1, 1e-2, 1e-3, 1e-4, 1e-5, 0.0]).repeat_interleave(H // 6 + 1)[:H]
    res = (-total + scales.double() * torch.randn(T, H, generator=gen).double()).to(td)
    w = (1.0 + 0.1 * torch.randn(H, generator=gen)).to(td)
    inp = wl.NormInputs(parts, res, w, T, H, W, dtype, wl.eps32(1e-6), False, True)
    check_norm(lib, inp, plan=plan)


@pytest.mark.parametrize("plan", NORM_PLANS)
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_fp8_rare_accuracy_paths(lib, plan, dtype):
    """Crafted rows that drive the FP8 variant's rare paths.
    row 0, elements 0-15: residual 1, partials k*tiny, -1, 0.  The fp32 sum
    1 + k*tiny is not exact, so the sums rounded down and up differ and the
    TwoSum recomputation must recover r = k*tiny (a plain fp32 sum gives 0).
    row 1, group 1: values near 1e-30 (bf16; zero in fp16) while the rest of
    the row is ordinary: the group scale falls below 2^-90 and the codes take
    the IEEE division.
    row 2, group 2: residual = -(sum of partials) exactly and weight -1: the
    group is all zeros (scale 0, codes 0) with signed-zero outputs.
    row 3: ordinary."""
    T, H, W = 4, 512, 3
    td = TD[dtype]
    tiny = 2.0 ** -30 if dtype == "bf16" else 2.0 ** -24
    gen = torch.Generator().manual_seed(4242 + plan)
    parts = [0.5 * torch.randn(T, H, generator=gen) for _ in range(W)]
    res = torch.randn(T, H, generator=gen)
    w = 1.0 + 0.1 * torch.randn(H, generator=gen)
    k = torch.arange(1, 17, dtype=torch.float32)
    res[0, :16], parts[0][0, :16], parts[1][0, :16], parts[2][0, :16] = 1.0, k * tiny, -1.0, 0.0
    for x in [res] + parts:
        x[1, 128:256] *= 1e-30
    g2 = slice(256, 384)
    for n, x in enumerate(parts):
        x[2, g2] = torch.randint(-8, 9, (128,), generator=gen).float() * (n + 1)
    res[2, g2] = -(parts[0][2, g2] + parts[1][2, g2] + parts[2][2, g2])
    w[g2] = -1.0
    parts = [x.to(td) for x in parts]
    inp = wl.NormInputs(parts, res.to(td), w.to(td), T, H, W, dtype, wl.eps32(1e-6), False, True)
    q, s, y, r = run_fp8(lib, inp, plan=plan)
    o = P.oracle_norm(inp)
    P.check_fp8(q, s, o["y"])
    P.check_y(y, o["y"], dtype)
    P.check_res(r, o["r"], dtype)
    exact = (k * tiny).to(td).view(torch.int16).numpy()
    assert np.array_equal(r[0, :16].astype(np.int16), exact), "TwoSum recovery of r = k*tiny"
    assert np.all(s[2, 2] == 0.0) and np.all(q[2, 256:384] & 0x7F == 0)
