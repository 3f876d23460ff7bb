"""torch.ops.ar_b200.*: registration, fake-tensor shape propagation and
argument checks (CPU), and on a GPU: identical results to the direct calls,
CUDA-graph capture, and torch.library.opcheck."""
import pytest
import torch
from torch._subclasses.fake_tensor import FakeTensorMode

import tensor_allreduce_residual_ar_b200 as ar  # noqa: F401  (registers the ops)
from tensor_allreduce_residual_ar_b200 import workloads as wl

OPS = torch.ops.ar_b200


def test_ops_are_registered_with_their_schemas():
    s = str(OPS.add_rmsnorm.default._schema)
    assert "Tensor[] partials, Tensor? residual, Tensor weight, float eps, bool gemma" in s
    assert s.endswith("-> (Tensor, Tensor)")
    assert str(OPS.add_rmsnorm_out_only.default._schema).endswith("-> Tensor")
    assert str(OPS.add_rmsnorm_fp8_group.default._schema).endswith("-> (Tensor, Tensor, Tensor, Tensor)")
    assert str(OPS.qk_norm_sharded.default._schema).endswith("-> (Tensor[], Tensor[])")


def test_fake_shapes_norm_and_fp8():
    with FakeTensorMode():
        parts = [torch.empty(2, 3, 5120, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
        res = torch.empty(2, 3, 5120, dtype=torch.bfloat16, device="cuda")
        w = torch.empty(5120, dtype=torch.bfloat16, device="cuda")
        y, r = OPS.add_rmsnorm(parts, res, w, 1e-6, True)
        assert y.shape == r.shape == (2, 3, 5120) and y.dtype == torch.bfloat16
        y2 = OPS.add_rmsnorm_out_only(parts, None, w, 1e-6, False)
        assert y2.shape == (2, 3, 5120)
        q, s, y3, r3 = OPS.add_rmsnorm_fp8_group(parts, res, w, 1e-6, False)
        assert q.shape == (2, 3, 5120) and q.dtype == torch.float8_e4m3fn
        assert s.shape == (2, 3, 40) and s.dtype == torch.float32
        assert y3.shape == r3.shape == (2, 3, 5120)


def test_tensor_parallel_ops_schemas_and_fake_shapes():
    s = str(OPS.tp_add_rmsnorm.default._schema)
    assert "Tensor partial, Tensor? residual, Tensor weight, float eps, bool gemma, SymInt comm" in s
    assert s.endswith("-> (Tensor, Tensor)")
    assert str(OPS.tp_add_rmsnorm_out_only.default._schema).endswith("-> Tensor")
    assert str(OPS.tp_add_rmsnorm_fp8_group.default._schema).endswith("-> (Tensor, Tensor, Tensor, Tensor)")
    with FakeTensorMode():
        p = torch.empty(5, 5120, dtype=torch.bfloat16, device="cuda")
        w = torch.empty(5120, dtype=torch.bfloat16, device="cuda")
        y, r = OPS.tp_add_rmsnorm(p, p, w, 1e-6, False, 3)
        assert y.shape == r.shape == (5, 5120)
        assert OPS.tp_add_rmsnorm_out_only(p, None, w, 1e-6, True, 3).shape == (5, 5120)
        q, sc, y2, r2 = OPS.tp_add_rmsnorm_fp8_group(p, p, w, 1e-6, False, 3)
        assert q.dtype == torch.float8_e4m3fn and sc.shape == (5, 40)
        with pytest.raises(ValueError):
            OPS.tp_add_rmsnorm(p, p[:, :4096], w, 1e-6, False, 3)
        qkv = torch.empty(9, 768 + 256, dtype=torch.bfloat16, device="cuda")     # W = 8 shard
        qw = torch.empty(6144, dtype=torch.bfloat16, device="cuda")
        kw = torch.empty(1024, dtype=torch.bfloat16, device="cuda")
        qo, ko = OPS.tp_qk_norm_sharded(qkv, qw, kw, 6144, 1024, 1e-6, 3)
        assert qo.shape == (9, 768) and ko.shape == (9, 128)
    assert str(OPS.tp_qk_norm_sharded.default._schema).endswith("-> (Tensor, Tensor)")


def test_fake_shapes_qk():
    with FakeTensorMode():
        qkv = [torch.empty(7, 768 + 256, dtype=torch.float16, device="cuda") for _ in range(8)]
        qw = torch.empty(6144, dtype=torch.float16, device="cuda")
        kw = torch.empty(1024, dtype=torch.float16, device="cuda")
        qo, ko = OPS.qk_norm_sharded(qkv, qw, kw, 6144, 1024, 1e-6)
        assert len(qo) == len(ko) == 8
        assert all(t.shape == (7, 768) for t in qo) and all(t.shape == (7, 128) for t in ko)
        assert qo[0].dtype == torch.float16


def test_fake_argument_checks():
    with FakeTensorMode():
        a = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
        w = torch.empty(64, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(ValueError):
            OPS.add_rmsnorm([a, torch.empty(4, 32, dtype=torch.bfloat16, device="cuda")], None, w, 1e-6, False)
        with pytest.raises(TypeError):
            OPS.add_rmsnorm([a], None, w.to(torch.float16), 1e-6, False)
        with pytest.raises(ValueError):
            OPS.add_rmsnorm_fp8_group([a], None, w, 1e-6, False)        # H = 64 < group 128
        qkv = [torch.empty(2, 64 + 64, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        with pytest.raises(ValueError):
            OPS.qk_norm_sharded(qkv, torch.empty(128, dtype=torch.bfloat16, device="cuda"),
                                torch.empty(64, dtype=torch.bfloat16, device="cuda"), 100, 64, 1e-6)


def test_cpu_tensors_are_rejected():
    a = torch.zeros(2, 64, dtype=torch.bfloat16)
    with pytest.raises(NotImplementedError):
        OPS.add_rmsnorm([a], None, torch.ones(64, dtype=torch.bfloat16), 1e-6, False)


# --------------------------------------------------------------------------- GPU

def _norm_inputs(T=33, dtype="bf16", fp8=False):
    inp = wl.make_norm_inputs(wl.FP8 if fp8 else wl.DECODE, T, dtype, seed=4242 + T)
    return ([p.cuda() for p in inp.partials], inp.residual.cuda(), inp.weight.cuda(), inp.eps,
            inp.gemma)


@pytest.mark.gpu
def test_ops_match_the_direct_calls(lib):
    parts, res, w, eps, gemma = _norm_inputs()
    y, r = OPS.add_rmsnorm(parts, res, w, eps, gemma)
    y0, r0 = torch.empty_like(res), torch.empty_like(res)
    lib.ar_add_rmsnorm(parts, res, w, y0, r0, eps=eps, gemma=gemma)
    assert torch.equal(y, y0) and torch.equal(r, r0)
    assert torch.equal(OPS.add_rmsnorm_out_only(parts, res, w, eps, gemma), y0)

    parts, res, w, eps, gemma = _norm_inputs(T=9, fp8=True)
    q, s, y, r = OPS.add_rmsnorm_fp8_group(parts, res, w, eps, gemma)
    q0 = torch.empty(res.shape, dtype=torch.uint8, device="cuda")
    s0 = torch.empty((res.shape[0], res.shape[1] // 128), dtype=torch.float32, device="cuda")
    y0, r0 = torch.empty_like(res), torch.empty_like(res)
    lib.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q0, s0, y0, r0, eps=eps, gemma=gemma)
    assert torch.equal(q.view(torch.uint8), q0) and torch.equal(s, s0)
    assert torch.equal(y, y0) and torch.equal(r, r0)

    inp = wl.make_qk_inputs(wl.QK, 64, seed=91)
    qkv = [x.cuda() for x in inp.qkv]
    qo, ko = OPS.qk_norm_sharded(qkv, inp.q_weight.cuda(), inp.k_weight.cuda(), inp.q_size,
                                 inp.kv_size, inp.eps)
    qs, ks = inp.q_size // inp.W, inp.kv_size // inp.W
    qo0 = [torch.empty((64, qs), dtype=torch.bfloat16, device="cuda") for _ in range(inp.W)]
    ko0 = [torch.empty((64, ks), dtype=torch.bfloat16, device="cuda") for _ in range(inp.W)]
    lib.qk_norm_sharded(qkv, inp.q_weight.cuda(), inp.k_weight.cuda(), qo0, ko0, inp.q_size,
                        inp.kv_size, eps=inp.eps)
    assert all(torch.equal(a, b) for a, b in zip(qo + ko, qo0 + ko0))


@pytest.mark.gpu
def test_ops_in_a_cuda_graph(lib):
    parts, res, w, eps, gemma = _norm_inputs(T=16)
    static = [p.clone() for p in parts]
    OPS.add_rmsnorm(static, res, w, eps, gemma)           # first call outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        y, r = OPS.add_rmsnorm(static, res, w, eps, gemma)
    for scale in (1.0, -0.5):
        for s_, p in zip(static, parts):
            s_.copy_(p * scale)
        g.replay()
        torch.cuda.synchronize()
        y0, r0 = OPS.add_rmsnorm(static, res, w, eps, gemma)
        assert torch.equal(y, y0) and torch.equal(r, r0)


@pytest.mark.gpu
def test_opcheck(lib):
    parts, res, w, eps, gemma = _norm_inputs(T=8)
    utils = ("test_schema", "test_faketensor")
    torch.library.opcheck(OPS.add_rmsnorm.default, (parts, res, w, eps, gemma), test_utils=utils)
    torch.library.opcheck(OPS.add_rmsnorm_out_only.default, (parts, None, w, eps, gemma), test_utils=utils)
    parts, res, w, eps, gemma = _norm_inputs(T=4, fp8=True)
    torch.library.opcheck(OPS.add_rmsnorm_fp8_group.default, (parts, res, w, eps, gemma), test_utils=utils)
    inp = wl.make_qk_inputs(wl.QK, 3, seed=5)
    torch.library.opcheck(OPS.qk_norm_sharded.default,
                          ([x.cuda() for x in inp.qkv], inp.q_weight.cuda(), inp.k_weight.cuda(),
                           inp.q_size, inp.kv_size, inp.eps), test_utils=utils)
