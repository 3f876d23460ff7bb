"""GPU parity of the multi-GPU form (all-reduce fused with add + RMSNorm, its
FP8 output, the sharded QK-norm) against the fp64 oracle.

On one GPU the W ranks run as a group: every rank's part in one cooperative
launch, each rank with its own device region, exchanging through the same
flags, staging slots and plain loads as the multi-GPU form (the kernels and
the protocol are the same code; only the region pointers differ).  The
world-size-1 rank form runs the multi-process launch path itself.  Every
rank's outputs must be bit-identical (an all-reduce replicates), match the
oracle on the W partials in rank order, and leave the guard bands intact."""
import numpy as np
import pytest
import torch

import parity as P
from tensor_allreduce_residual_ar_b200 import comm as C
from tensor_allreduce_residual_ar_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD = 512
SENT16 = 0x5A5A
TD = {"bf16": torch.bfloat16, "fp16": torch.float16}


class Guarded:
    def __init__(self, shape, dtype, sentinel):
        n = int(np.prod(shape))
        raw = torch.int16 if dtype in (torch.bfloat16, torch.float16) else dtype
        self.buf = torch.full((n + GUARD,), sentinel, dtype=raw, device="cuda")
        self.n, self.sentinel = n, sentinel
        self.view = self.buf[:n].view(dtype).view(*shape) if raw != dtype else self.buf[:n].view(*shape)

    def guard_ok(self):
        return bool((self.buf[self.n:] == self.sentinel).all().item())


def run_group_norm(g, inp, algo, write_res=True, residual=True):
    W, T, H = inp.W, inp.T, inp.H
    td = TD[inp.dtype]
    parts = [p.to("cuda") for p in inp.partials]
    res = [inp.residual.to("cuda") for _ in range(W)] if residual else None
    outs = [Guarded((T, H), td, SENT16) for _ in range(W)]
    routs = [Guarded((T, H), td, SENT16) for _ in range(W)] if write_res else None
    g.allreduce_add_rmsnorm(parts, res, inp.weight.to("cuda"), [o.view for o in outs],
                            [r.view for r in routs] if routs else None, eps=inp.eps,
                            gemma=inp.gemma, algo=algo)
    torch.cuda.synchronize()
    assert g.status() == 0
    for b in outs + (routs or []):
        assert b.guard_ok()
    ys = [P.to_bits(o.view) for o in outs]
    rs = [P.to_bits(r.view) for r in routs] if routs else None
    return ys, rs


def check_group_norm(g, inp, algo, write_res=True, residual=True):
    ys, rs = run_group_norm(g, inp, algo, write_res, residual)
    for w in range(1, inp.W):
        assert np.array_equal(ys[w], ys[0]), f"rank {w}'s y differs from rank 0's"
        if rs is not None:
            assert np.array_equal(rs[w], rs[0]), f"rank {w}'s residual_out differs"
    ref = inp if residual else wl.NormInputs(inp.partials, None, inp.weight, inp.T, inp.H, inp.W,
                                             inp.dtype, inp.eps, inp.gemma, write_res)
    o = P.oracle_norm(ref)
    st = P.check_y(ys[0], o["y"], inp.dtype)
    if inp.dtype == "bf16":
        assert st["ulp_clause"] == 0
    if rs is not None:
        P.check_res(rs[0], o["r"], inp.dtype)
    return ys[0]


CASES = [  # (W, T, H, dtype, gemma)
    (2, 1, 8192, "bf16", True), (4, 5, 8192, "fp16", True), (8, 80, 8192, "bf16", True),
    (4, 33, 4096, "bf16", False), (3, 7, 1000, "bf16", False), (8, 300, 4096, "bf16", False),
    (16, 9, 2048, "fp16", False), (5, 2, 64, "bf16", True),
]


@pytest.mark.parametrize("algo", ["oneshot", "twoshot"])
@pytest.mark.parametrize("W,T,H,dtype,gemma", CASES)
def test_group_allreduce_add_rmsnorm(lib, algo, W, T, H, dtype, gemma):
    inp = wl.make_norm_inputs(wl.DECODE, T, dtype, W=W, H=H, seed=4000 + W * 100 + T + H)
    inp.gemma = gemma
    g = C.CommGroup(W, T * H)
    try:
        check_group_norm(g, inp, algo)
        check_group_norm(g, inp, algo, write_res=False)            # dead residual
        check_group_norm(g, inp, algo, residual=False)             # no residual
    finally:
        g.close()


def test_group_prefill_shape_two_shot(lib):
    """The prefill configuration's shape over 8 ranks (T=8192, H=4096, one
    partial per rank, dead residual), two-shot: sampled rows checked."""
    inp = wl.make_norm_inputs(wl.PREFILL, 8192, seed=4242)
    g = C.CommGroup(8, 8192 * 4096)
    try:
        ys, _ = run_group_norm(g, inp, "twoshot", write_res=False)
    finally:
        g.close()
    for w in range(1, 8):
        assert np.array_equal(ys[w], ys[0])
    rows = np.unique(np.concatenate([[0, 1023, 1024, 8191],
                                     np.random.default_rng(1).choice(8192, 60, replace=False)]))
    o = P.oracle_norm(inp, rows=rows)
    P.check_y(ys[0][rows], o["y"], "bf16")


@pytest.mark.parametrize("plan", [1, 3, 4, 5, 9, 10])
def test_one_shot_equals_single_gpu_call(lib, plan):
    """With the same plan, the one-shot exchange computes exactly what the
    single-GPU call computes from the W partials in rank order."""
    W, T, H = 4, 24, 8192
    inp = wl.make_norm_inputs(wl.DECODE, T, "bf16", W=W, H=H, seed=77 + plan)
    assert lib.ar_plan_force(0, plan) == 0
    g = C.CommGroup(W, T * H)
    try:
        ys, rs = run_group_norm(g, inp, "oneshot")
    finally:
        g.close()
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    rout = torch.empty_like(out)
    lib.ar_add_rmsnorm([p.cuda() for p in inp.partials], inp.residual.cuda(), inp.weight.cuda(), out,
                       rout, eps=inp.eps, gemma=inp.gemma)
    torch.cuda.synchronize()
    assert np.array_equal(ys[0], P.to_bits(out))
    assert np.array_equal(rs[0], P.to_bits(rout))


@pytest.mark.parametrize("algo", ["oneshot", "twoshot"])
@pytest.mark.parametrize("W,T,H,residual", [(4, 1, 5120, True), (4, 67, 5120, True),
                                            (2, 130, 2048, False), (8, 17, 1024, True)])
def test_group_fp8(lib, algo, W, T, H, residual):
    inp = wl.make_norm_inputs(wl.FP8, T, W=W, H=H, residual=residual, seed=5000 + T + H + W)
    G = H // 128
    g = C.CommGroup(W, T * H)
    try:
        parts = [p.cuda() for p in inp.partials]
        res = [inp.residual.cuda() for _ in range(W)] if residual else None
        q = [Guarded((T, H), torch.uint8, 0xA5) for _ in range(W)]
        s = [Guarded((T, G), torch.float32, -7.0) for _ in range(W)]
        y = [Guarded((T, H), torch.bfloat16, SENT16) for _ in range(W)]
        r = [Guarded((T, H), torch.bfloat16, SENT16) for _ in range(W)]
        g.allreduce_add_rmsnorm_quant_fp8_group(parts, res, inp.weight.cuda(), [b.view for b in q],
                                                [b.view for b in s], [b.view for b in y],
                                                [b.view for b in r], eps=inp.eps, algo=algo)
        torch.cuda.synchronize()
        assert g.status() == 0
    finally:
        g.close()
    for b in q + s + y + r:
        assert b.guard_ok()
    qs = [b.view.cpu().numpy() for b in q]
    ss = [b.view.cpu().numpy() for b in s]
    for w in range(1, W):
        assert np.array_equal(qs[w], qs[0]) and np.array_equal(ss[w], ss[0])
        assert np.array_equal(P.to_bits(y[w].view), P.to_bits(y[0].view))
    o = P.oracle_norm(inp)
    P.check_fp8(qs[0], ss[0], o["y"])
    P.check_y(P.to_bits(y[0].view), o["y"], "bf16")
    P.check_res(P.to_bits(r[0].view), o["r"], "bf16")


@pytest.mark.parametrize("inplace", [False, True])
@pytest.mark.parametrize("T,W,q_size,kv_size,dtype", [(1, 8, 6144, 1024, "bf16"),
                                                      (64, 8, 6144, 1024, "bf16"),
                                                      (300, 8, 6144, 1024, "fp16"),
                                                      (9, 2, 256, 128, "bf16"),
                                                      (5, 16, 2048, 128, "bf16")])
def test_group_qk(lib, inplace, T, W, q_size, kv_size, dtype):
    inp = wl.make_qk_inputs(wl.QK, T, dtype, W=W, q_size=q_size, kv_size=kv_size, seed=600 + T + W)
    qs, ks = q_size // W, kv_size // W
    td = TD[dtype]
    qkv = [x.to("cuda").clone() for x in inp.qkv]
    v_before = [x[:, qs + ks:].clone() for x in qkv]
    if inplace:
        qo = [x[:, :qs] for x in qkv]
        ko = [x[:, qs:qs + ks] for x in qkv]
        gq = gk = None
    else:
        gq = [Guarded((T, qs), td, SENT16) for _ in range(W)]
        gk = [Guarded((T, ks), td, SENT16) for _ in range(W)]
        qo, ko = [b.view for b in gq], [b.view for b in gk]
    g = C.CommGroup(W, max(8, 4 * T))
    try:
        g.qk_norm_sharded(qkv, inp.q_weight.cuda(), inp.k_weight.cuda(), qo, ko, q_size, kv_size,
                          eps=inp.eps)
        torch.cuda.synchronize()
        assert g.status() == 0
    finally:
        g.close()
    q64, k64 = P.oracle_qk(inp)
    for w in range(W):
        P.check_y(P.to_bits(qo[w].contiguous()), q64[w], dtype, f"q[{w}]")
        P.check_y(P.to_bits(ko[w].contiguous()), k64[w], dtype, f"k[{w}]")
        assert torch.equal(qkv[w][:, qs + ks:], v_before[w]), "v must not be modified"
    if gq:
        assert all(b.guard_ok() for b in gq + gk)


def test_group_many_calls_alternate_slots(lib):
    """One group, a run of calls with changing T, algorithm and form: the
    per-call epoch, the alternating slots and the per-CTA flags stay in step
    across calls of different grid sizes."""
    W, H = 4, 4096
    g = C.CommGroup(W, 256 * H)
    try:
        for i, (T, algo) in enumerate([(1, "oneshot"), (256, "twoshot"), (3, "twoshot"),
                                       (100, "oneshot"), (256, "oneshot"), (2, "twoshot"),
                                       (77, "twoshot"), (1, "oneshot")]):
            inp = wl.make_norm_inputs(wl.DECODE, T, "bf16", W=W, H=H, seed=900 + i)
            check_group_norm(g, inp, algo)
        T = 48
        inp = wl.make_qk_inputs(wl.QK, T, W=W, q_size=512, kv_size=256, seed=901)
        qo = [torch.empty((T, 128), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
        ko = [torch.empty((T, 64), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
        g.qk_norm_sharded([x.cuda() for x in inp.qkv], inp.q_weight.cuda(), inp.k_weight.cuda(),
                          qo, ko, 512, 256, eps=inp.eps)
        torch.cuda.synchronize()
        q64, k64 = P.oracle_qk(inp)
        for w in range(W):
            P.check_y(P.to_bits(qo[w]), q64[w], "bf16")
            P.check_y(P.to_bits(ko[w]), k64[w], "bf16")
        inp = wl.make_norm_inputs(wl.DECODE, 64, "fp16", W=W, H=H, seed=902)
        check_group_norm(g, inp, "twoshot")
    finally:
        g.close()


def test_withheld_arrival_times_out_and_is_reported(lib):
    """One rank publishes no arrival: every other rank's bounded wait runs
    out, the launch still finishes, the status says AR_ETIMEDOUT (5); a new
    group then computes correctly."""
    W, T, H = 4, 16, 2048
    inp = wl.make_norm_inputs(wl.DECODE, T, "bf16", W=W, H=H, seed=31)
    g = C.CommGroup(W, T * H)
    try:
        g.set_timeout(0.05)
        g.test_withhold(2)
        parts = [p.cuda() for p in inp.partials]
        outs = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
        g.allreduce_add_rmsnorm(parts, None, inp.weight.cuda(), outs, None, eps=inp.eps, algo="oneshot")
        assert g.status(clear=True) == 5
        assert g.status() == 0
    finally:
        g.close()
    g = C.CommGroup(W, T * H)
    try:
        check_group_norm(g, inp, "oneshot")
        check_group_norm(g, inp, "twoshot")
    finally:
        g.close()


def test_rank_form_world_one(lib):
    """The multi-process launch path with a single rank: the sum over ranks
    is the rank's own partial."""
    T, H = 40, 8192
    inp = wl.make_norm_inputs(wl.DECODE, T, "bf16", W=1, H=H, seed=55)
    c = C.Comm(T * H)
    try:
        assert c.world == 1
        for algo in ("oneshot", "twoshot"):
            out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
            rout = torch.empty_like(out)
            c.allreduce_add_rmsnorm(inp.partials[0].cuda(), inp.residual.cuda(), inp.weight.cuda(), out,
                                    rout, eps=inp.eps, gemma=inp.gemma, algo=algo)
            torch.cuda.synchronize()
            o = P.oracle_norm(inp)
            P.check_y(P.to_bits(out), o["y"], "bf16")
            P.check_res(P.to_bits(rout), o["r"], "bf16")
        assert c.status() == 0
    finally:
        c.close()


def test_rank_form_graph_replays_advance_the_epoch(lib):
    """Captured in a CUDA graph, each replay advances the device-side epoch
    (no host state in the launch), so replays keep alternating slots and
    stay correct."""
    T, H = 8, 4096
    c = C.Comm(T * H)
    try:
        part = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        res = torch.empty_like(part)
        w = torch.empty((H,), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(part)
        inp0 = wl.make_norm_inputs(wl.TINY, T, W=1, H=H, seed=1)
        part.copy_(inp0.partials[0]); res.copy_(inp0.residual); w.copy_(inp0.weight)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            c.allreduce_add_rmsnorm(part, res, w, out, None, eps=inp0.eps)   # outside capture first
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(graph, stream=s):
                c.allreduce_add_rmsnorm(part, res, w, out, None, eps=inp0.eps)
        for i in range(3):
            inp = wl.make_norm_inputs(wl.TINY, T, W=1, H=H, seed=10 + i)
            part.copy_(inp.partials[0]); res.copy_(inp.residual); w.copy_(inp.weight)
            graph.replay()
            torch.cuda.synchronize()
            P.check_y(P.to_bits(out), P.oracle_norm(inp)["y"], "bf16")
        del graph
        assert c.status() == 0
    finally:
        c.close()


def test_crossover_tuning_sets_the_communicator(lib):
    """The collective crossover measurement runs both forms and sets the
    one-shot limit to the size the measured rows give (world size 1 here: both
    forms are the rank's own sum, and the automatic choice stays one-shot at
    any size because one rank has nothing to exchange)."""
    c = C.Comm(512 * 4096)
    try:
        limit = c.tune_oneshot_max(H=4096, Ts=(1, 8, 64, 512), iters=5)
        assert [r[0] for r in c.crossover_us] == [1, 8, 64, 512]
        assert all(r[1] > 0 and r[2] > 0 for r in c.crossover_us)
        assert limit == C.oneshot_limit(c.crossover_us, 4096)
        for T in (1, 8, 64, 512):
            assert c.algo(T, 4096) == "oneshot"
        assert c.status() == 0
    finally:
        c.close()
