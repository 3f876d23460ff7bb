"""The graph rewrite that routes unfused all-reduce + add + RMSNorm subgraphs
to torch.ops.ar_b200.*: how many times each form fires on toy programs
(CPU, tracing only), that nothing unrecognised is touched, and (GPU) that
the rewritten program's outputs match the fp64 oracle."""
import operator

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from tensor_allreduce_residual_ar_b200 import fx_patterns as FX


def targets(gm):
    return [n.target for n in gm.graph.nodes if n.op == "call_function"]


def fused_ops(gm):
    return [t for t in targets(gm) if str(t).startswith("ar_b200.")]


class TwoOutput(torch.nn.Module):
    def forward(self, p0, p1, p2, res, w):
        r = (p0 + p1 + p2) + res
        y = F.rms_norm(r, (r.shape[-1],), w, 1e-6)
        return y * 2, r


class OutOnly(torch.nn.Module):
    def forward(self, p0, p1, res, w):
        r = res + (p0 + p1)
        return F.rms_norm(r, (r.shape[-1],), w, 1e-5)


class NoResidual(torch.nn.Module):
    def forward(self, p0, p1, p2, p3, w):
        s = FX.all_reduce_sum_reference([p0, p1, p2, p3])
        return F.rms_norm(s, (s.shape[-1],), w, 1e-6)


class NoResidualTwoAdds(torch.nn.Module):
    def forward(self, p0, p1, w):
        s = p0 + p1
        return F.rms_norm(s, (s.shape[-1],), w, 1e-6), s


class Gemma(torch.nn.Module):
    def forward(self, p0, p1, res, w):
        r = FX.all_reduce_sum_reference([p0, p1]) + res
        return F.rms_norm(r, (r.shape[-1],), None, 1e-6) * (1 + w), r


class Fp8(torch.nn.Module):
    def forward(self, p0, p1, p2, p3, res, w):
        r = FX.all_reduce_sum_reference([p0, p1, p2, p3]) + res
        y = F.rms_norm(r, (r.shape[-1],), w, 1e-6)
        q, s = FX.quant_fp8_group_reference(y)
        return q, s, y, r          # the 16-bit y kept for a second consumer


class TwoLayers(torch.nn.Module):
    """Two sub-layers: the first's residual result feeds the second."""

    def forward(self, a0, a1, b0, b1, res, w1, w2):
        r1 = FX.all_reduce_sum_reference([a0, a1]) + res
        y1 = F.rms_norm(r1, (r1.shape[-1],), w1, 1e-6)
        r2 = FX.all_reduce_sum_reference([b0 * y1, b1]) + r1
        y2 = F.rms_norm(r2, (r2.shape[-1],), w2, 1e-6)
        return y2


COMM = 7      # a communicator id as the traced programs carry it (registered only on the GPU)


class TpTwoOutput(torch.nn.Module):
    def forward(self, p, res, w):
        r = FX.tp_all_reduce_reference(p, COMM) + res
        return F.rms_norm(r, (r.shape[-1],), w, 1e-6), r


class TpOutOnly(torch.nn.Module):
    def forward(self, p, res, w):
        r = res + FX.tp_all_reduce_reference(p, COMM)
        return F.rms_norm(r, (r.shape[-1],), w, 1e-5)


class TpNoResidual(torch.nn.Module):
    def forward(self, p, w):
        s = FX.tp_all_reduce_reference(p, COMM)
        return F.rms_norm(s, (s.shape[-1],), w, 1e-6)


class TpGemma(torch.nn.Module):
    def forward(self, p, res, w):
        r = FX.tp_all_reduce_reference(p, COMM) + res
        return F.rms_norm(r, (r.shape[-1],), None, 1e-6) * (1 + w), r


class TpFp8(torch.nn.Module):
    def forward(self, p, res, w):
        r = FX.tp_all_reduce_reference(p, COMM) + res
        y = F.rms_norm(r, (r.shape[-1],), w, 1e-6)
        q, s = FX.quant_fp8_group_reference(y)
        return q, s, y, r


class TpSumReadElsewhere(torch.nn.Module):
    """The all-reduced sum is read again besides the residual add: the add +
    norm is still fused (the sum is not a private intermediate of it, so it
    stays), exactly like a shared partial sum on one GPU."""

    def forward(self, p, res, w):
        s = FX.tp_all_reduce_reference(p, COMM)
        r = s + res
        return F.rms_norm(r, (r.shape[-1],), w, 1e-6), s * 2


class NotASum(torch.nn.Module):
    def forward(self, x, res, w):
        r = x * res
        return F.rms_norm(r, (r.shape[-1],), w, 1e-6)


class PartialSumUsedElsewhere(torch.nn.Module):
    def forward(self, p0, p1, p2, w):
        s01 = p0 + p1                    # read again below: not a private chain
        r = s01 + p2
        return F.rms_norm(r, (r.shape[-1],), w, 1e-6), s01 * 3


class ReaderBeforeWeight(torch.nn.Module):
    def forward(self, p0, p1, res, w0):
        r = FX.all_reduce_sum_reference([p0, p1]) + res
        z = r * 2                        # reads r before the weight exists
        w = w0 + 0.5
        return F.rms_norm(r, (r.shape[-1],), w, 1e-6), z


def fuse(mod):
    gm = torch.fx.symbolic_trace(mod)
    return gm, FX.fuse_allreduce_rmsnorm(gm)


@pytest.mark.parametrize("mod,want,op", [
    (TwoOutput(), {"two_output": 1}, "add_rmsnorm"),
    (OutOnly(), {"out_only": 1}, "add_rmsnorm_out_only"),
    (NoResidual(), {"out_only": 1, "no_residual": 1}, "add_rmsnorm_out_only"),
    (NoResidualTwoAdds(), {"two_output": 1, "no_residual": 1}, "add_rmsnorm"),
    (Gemma(), {"two_output": 1, "gemma": 1}, "add_rmsnorm"),
    (Fp8(), {"fp8": 1}, "add_rmsnorm_fp8_group"),
])
def test_each_form_fires_once(mod, want, op):
    gm, c = fuse(mod)
    full = {"two_output": 0, "out_only": 0, "no_residual": 0, "fp8": 0, "gemma": 0, "tp": 0, **want}
    assert c == full
    ops = fused_ops(gm)
    assert [str(t).split(".")[1] for t in ops] == [op]
    left = targets(gm)
    assert not any(t in FX._NORMS for t in left), "the unfused norm is gone"
    assert FX.quant_fp8_group_reference not in left and FX.all_reduce_sum_reference not in left
    assert not any(t in FX._ADDS for t in left), "the partial sum and the residual add are gone"


@pytest.mark.parametrize("mod,want,op", [
    (TpTwoOutput(), {"two_output": 1}, "tp_add_rmsnorm"),
    (TpOutOnly(), {"out_only": 1}, "tp_add_rmsnorm_out_only"),
    (TpNoResidual(), {"out_only": 1, "no_residual": 1}, "tp_add_rmsnorm_out_only"),
    (TpGemma(), {"two_output": 1, "gemma": 1}, "tp_add_rmsnorm"),
    (TpFp8(), {"fp8": 1}, "tp_add_rmsnorm_fp8_group"),
])
def test_tensor_parallel_forms_route_to_the_communicator(mod, want, op):
    gm, c = fuse(mod)
    full = {"two_output": 0, "out_only": 0, "no_residual": 0, "fp8": 0, "gemma": 0, "tp": 1, **want}
    assert c == full
    ops = fused_ops(gm)
    assert [str(t).split(".")[1] for t in ops] == [op]
    node = [n for n in gm.graph.nodes if str(n.target).startswith("ar_b200.")][0]
    assert node.args[-1] == COMM and node.args[0].op == "placeholder"   # this rank's partial, the id
    left = targets(gm)
    assert FX.tp_all_reduce_reference not in left
    assert not any(t in FX._NORMS for t in left)


def test_tensor_parallel_sum_read_elsewhere():
    gm, c = fuse(TpSumReadElsewhere())
    # the all-reduce is not private to the add + norm: the add is fused as
    # the sum of two plain terms (s and res) and the all-reduce stays
    assert c["tp"] == 0 and c["two_output"] + c["out_only"] == 1
    assert FX.tp_all_reduce_reference in targets(gm)


class TpTwoSublayers(torch.nn.Module):
    """A tensor-parallel decoder layer's two norm sites: the attention
    output's all-reduce + residual + RMSNorm (two outputs: the residual
    stream continues), then the MLP's (output only, the layer's last)."""

    def __init__(self, H=64):
        super().__init__()
        self.proj_a = torch.nn.Linear(H, H, bias=False)
        self.proj_b = torch.nn.Linear(H, H, bias=False)

    def forward(self, x, res, w1, w2):
        r1 = FX.tp_all_reduce_reference(self.proj_a(x), COMM) + res
        y1 = F.rms_norm(r1, (r1.shape[-1],), w1, 1e-6)
        r2 = FX.tp_all_reduce_reference(self.proj_b(y1), COMM) + r1
        return F.rms_norm(r2, (r2.shape[-1],), w2, 1e-6)


def test_tensor_parallel_two_sublayers():
    gm, c = fuse(TpTwoSublayers())
    assert c["tp"] == 2 and c["two_output"] == 1 and c["out_only"] == 1
    assert [str(t).split(".")[1] for t in fused_ops(gm)] == ["tp_add_rmsnorm", "tp_add_rmsnorm_out_only"]
    assert FX.tp_all_reduce_reference not in targets(gm)
    # the projections (call_module) are untouched
    assert sum(n.op == "call_module" for n in gm.graph.nodes) == 2


def test_two_layers_chain():
    gm, c = fuse(TwoLayers())
    assert c["two_output"] == 1 and c["out_only"] == 1
    assert len(fused_ops(gm)) == 2


@pytest.mark.parametrize("mod", [NotASum(), ReaderBeforeWeight()])
def test_unrecognised_graphs_are_left_alone(mod):
    gm, c = fuse(mod)
    before = torch.fx.symbolic_trace(mod)
    assert c == {"two_output": 0, "out_only": 0, "no_residual": 0, "fp8": 0, "gemma": 0, "tp": 0}
    assert targets(gm) == targets(before)


def test_shared_partial_sum_stays():
    """p0 + p1 is read elsewhere, so it is not a private part of the sum: the
    norm's input (p0 + p1) + p2 is fused as the sum of two terms, (p0 + p1)
    and p2, and p0 + p1 itself stays for its other reader."""
    gm, c = fuse(PartialSumUsedElsewhere())
    assert c["out_only"] == 1 and c["no_residual"] == 1
    assert targets(gm).count(operator.add) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("mod_cls,W,has_res", [(TwoOutput, 3, True), (OutOnly, 2, True),
                                                (NoResidual, 4, False), (Gemma, 2, True),
                                                (Fp8, 4, True), (NoResidualTwoAdds, 2, False)])
def test_rewritten_program_matches_oracle(lib, mod_cls, W, has_res):
    import parity as P
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    T, H = 37, 1024
    inp = wl.make_norm_inputs(wl.FP8, T, W=W, H=H, residual=has_res, seed=7100 + W)
    gemma = mod_cls is Gemma
    inp.gemma = gemma
    gm, c = fuse(mod_cls())
    assert sum(c[k] for k in ("two_output", "out_only", "fp8")) == 1
    args = [p.cuda() for p in inp.partials] + ([inp.residual.cuda()] if has_res else []) + \
        [inp.weight.cuda()]
    if mod_cls is OutOnly:
        args = [args[0], args[1], args[2], args[3]]
    out = gm(*args)
    torch.cuda.synchronize()
    outs = out if isinstance(out, tuple) else (out,)
    eps = {OutOnly: wl.eps32(1e-5)}.get(mod_cls, wl.eps32(1e-6))
    ref = wl.NormInputs(inp.partials, inp.residual if has_res else None, inp.weight, T, H, W, "bf16",
                        eps, gemma, True)
    o = P.oracle_norm(ref)
    if mod_cls is Fp8:
        q, s, y, r = outs
        P.check_fp8(q.view(torch.uint8).cpu().numpy(), s.cpu().numpy(), o["y"])
        P.check_y(P.to_bits(y), o["y"], "bf16")
        P.check_res(P.to_bits(r), o["r"], "bf16")
        return
    y = outs[0] / 2 if mod_cls is TwoOutput else outs[0]
    P.check_y(P.to_bits(y.contiguous()), o["y"], "bf16")
    if len(outs) > 1:
        P.check_res(P.to_bits(outs[1]), o["r"], "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("mod_cls,has_res", [(TpTwoOutput, True), (TpOutOnly, True), (TpNoResidual, False),
                                             (TpGemma, True), (TpFp8, True)])
def test_tensor_parallel_rewrite_matches_oracle(lib, mod_cls, has_res):
    """The rewritten tensor-parallel programs on a world-size-1 communicator
    (the all-reduce of one rank's partial is the partial itself) against the
    oracle; the operator passes torch.library.opcheck."""
    import parity as P
    from tensor_allreduce_residual_ar_b200 import comm as C
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    T, H = 37, 1024
    c = C.Comm(T * H)
    C._REGISTRY[COMM] = c          # the id the traced programs carry
    try:
        inp = wl.make_norm_inputs(wl.FP8, T, W=1, H=H, residual=has_res, seed=7300 + has_res)
        gemma = mod_cls is TpGemma
        inp.gemma = gemma
        gm, cnt = fuse(mod_cls())
        assert cnt["tp"] == 1
        args = [inp.partials[0].cuda()] + ([inp.residual.cuda()] if has_res else []) + [inp.weight.cuda()]
        eps = {TpOutOnly: wl.eps32(1e-5)}.get(mod_cls, wl.eps32(1e-6))
        ref = wl.NormInputs(inp.partials, inp.residual if has_res else None, inp.weight, T, H, 1, "bf16",
                            eps, gemma, True)
        o = P.oracle_norm(ref)
        for prog in (gm,):
            out = prog(*args)
            torch.cuda.synchronize()
            outs = out if isinstance(out, tuple) else (out,)
            if mod_cls is TpFp8:
                q, s, y, r = outs
                P.check_fp8(q.view(torch.uint8).cpu().numpy(), s.cpu().numpy(), o["y"])
                P.check_y(P.to_bits(y), o["y"], "bf16")
                P.check_res(P.to_bits(r), o["r"], "bf16")
                continue
            P.check_y(P.to_bits(outs[0].contiguous()), o["y"], "bf16")
            if len(outs) > 1:
                P.check_res(P.to_bits(outs[1]), o["r"], "bf16")
        if mod_cls is TpTwoOutput:
            torch.library.opcheck(torch.ops.ar_b200.tp_add_rmsnorm.default,
                                  (args[0], args[1], args[2], 1e-6, False, COMM))
    finally:
        C._REGISTRY.pop(COMM, None)
        c.close()


@pytest.mark.gpu
def test_tensor_parallel_qk_operator_matches_oracle(lib):
    """torch.ops.ar_b200.tp_qk_norm_sharded on a world-size-1 communicator
    (the rank's shard is the whole q and k) against the oracle."""
    import parity as P
    from tensor_allreduce_residual_ar_b200 import comm as C
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    T = 33
    inp = wl.make_qk_inputs(wl.QK, T, "bf16", W=1, q_size=6144, kv_size=1024, seed=7400)
    c = C.Comm(T * (6144 + 2 * 1024))
    cid = C.register(c)
    try:
        qo, ko = torch.ops.ar_b200.tp_qk_norm_sharded(inp.qkv[0].cuda(), inp.q_weight.cuda(),
                                                      inp.k_weight.cuda(), 6144, 1024, 1e-6, cid)
        torch.cuda.synchronize()
        q64, k64 = P.oracle_qk(inp)
        P.check_y(P.to_bits(qo), q64[0], "bf16")
        P.check_y(P.to_bits(ko), k64[0], "bf16")
    finally:
        C.unregister(cid)
        c.close()


@pytest.mark.gpu
def test_tensor_parallel_operator_in_a_cuda_graph(lib):
    """The tensor-parallel operator captured in a CUDA graph on a world-size-1
    communicator: replays give the eager call's bits (new inputs copied into
    the captured buffers between replays)."""
    from tensor_allreduce_residual_ar_b200 import comm as C
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    T, H = 24, 2048
    c = C.Comm(T * H)
    cid = C.register(c)
    try:
        ins = [wl.make_norm_inputs(wl.DECODE, T, "bf16", W=1, H=H, seed=7500 + i) for i in range(3)]
        p = ins[0].partials[0].cuda()
        res = ins[0].residual.cuda()
        w = ins[0].weight.cuda()
        op = torch.ops.ar_b200.tp_add_rmsnorm
        op(p, res, w, 1e-6, True, cid)                     # first call outside capture
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                y, r = op(p, res, w, 1e-6, True, cid)
        for inp in ins[1:]:
            p.copy_(inp.partials[0])
            res.copy_(inp.residual)
            g.replay()
            torch.cuda.synchronize()
            y0, r0 = op(p.clone(), res.clone(), w, 1e-6, True, cid)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), y0.view(torch.int16))
            assert torch.equal(r.view(torch.int16), r0.view(torch.int16))
        del g
    finally:
        C.unregister(cid)
        c.close()
