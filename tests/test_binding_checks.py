"""The Python binding rejects bad tensors before anything reaches the library.

A host tensor's data pointer, a buffer on another device or a buffer shorter
than the call implies would reach a kernel as an illegal address, so the
binding checks every tensor (type, dtype, shape, contiguity, device) first.
These tests run on a CPU-only host: the library loader is replaced by one
that fails the test, which proves that every rejection happens before it."""
import pytest
import torch

from tensor_allreduce_residual_ar_b200 import binding as B


@pytest.fixture(autouse=True)
def _no_library(monkeypatch):
    def boom():
        raise AssertionError("the library was reached before the arguments were rejected")
    monkeypatch.setattr(B, "load_library", boom)


def norm_args(T=4, H=64, W=3, dtype=torch.bfloat16):
    parts = [torch.zeros(T, H, dtype=dtype) for _ in range(W)]
    return parts, torch.zeros(T, H, dtype=dtype), torch.ones(H, dtype=dtype), \
        torch.empty(T, H, dtype=dtype), torch.empty(T, H, dtype=dtype)


def test_host_tensors_are_rejected():
    parts, res, w, out, rout = norm_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.ar_add_rmsnorm(parts, res, w, out, rout)


@pytest.mark.parametrize("which", ["partial", "residual", "out", "residual_out"])
def test_short_or_misshaped_buffers(which):
    parts, res, w, out, rout = norm_args()
    short = torch.zeros(3, 64, dtype=torch.bfloat16)
    if which == "partial":
        parts[2] = short
    elif which == "residual":
        res = short
    elif which == "out":
        out = short
    else:
        rout = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.ar_add_rmsnorm(parts, res, w, out, rout)


def test_mixed_dtypes():
    parts, res, w, out, rout = norm_args()
    parts[1] = parts[1].half()
    with pytest.raises(TypeError, match="dtype"):
        B.ar_add_rmsnorm(parts, res, w, out, rout)
    parts, res, w, out, rout = norm_args()
    with pytest.raises(TypeError, match="dtype"):
        B.ar_add_rmsnorm(parts, res, w, out.half(), rout)
    with pytest.raises(TypeError):
        B.ar_add_rmsnorm([p.float() for p in parts], res.float(), w.float(), out.float())


def test_non_contiguous_and_bad_weight():
    parts, res, w, out, rout = norm_args(H=64)
    wide = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="contiguous"):
        B.ar_add_rmsnorm(parts, wide[:, ::2], w, out, rout)
    with pytest.raises(ValueError, match="weight"):
        B.ar_add_rmsnorm(parts, res, torch.ones(2, 32, dtype=torch.bfloat16), out, rout)
    with pytest.raises(TypeError):
        B.ar_add_rmsnorm(parts, res, w, None)
    with pytest.raises(TypeError):
        B.ar_add_rmsnorm([], res, w, out)
    with pytest.raises(ValueError, match="at most"):
        B.ar_add_rmsnorm(parts * 6, res, w, out)
    with pytest.raises(TypeError):
        B.ar_add_rmsnorm([parts[0], parts[1].numpy()], res, w, out)


def test_fp8_outputs_checked():
    parts, res, w, out, rout = norm_args(H=256)
    q = torch.empty(4, 256, dtype=torch.uint8)
    s = torch.empty(4, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q, s, out, rout)
    with pytest.raises(TypeError, match="out_fp8"):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q.to(torch.int16), s, out, rout)
    with pytest.raises(TypeError, match="scales"):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q, s.double(), out, rout)
    with pytest.raises(ValueError):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q[:3], s, out, rout)
    with pytest.raises(ValueError, match="scales"):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q, torch.empty(4, 1), out, rout)
    with pytest.raises(ValueError):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, q, s, out[:2], rout)
    with pytest.raises(TypeError):
        B.ar_add_rmsnorm_quant_fp8_group(parts, res, w, None, s)


def qk_args(T=3, W=2, q_size=32, kv_size=16):
    qs, ks = q_size // W, kv_size // W
    qkv = [torch.zeros(T, qs + 2 * ks, dtype=torch.bfloat16) for _ in range(W)]
    return (qkv, torch.ones(q_size, dtype=torch.bfloat16), torch.ones(kv_size, dtype=torch.bfloat16),
            [torch.empty(T, qs, dtype=torch.bfloat16) for _ in range(W)],
            [torch.empty(T, ks, dtype=torch.bfloat16) for _ in range(W)])


def test_qk_checks():
    qkv, qw, kw, qo, ko = qk_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.qk_norm_sharded(qkv, qw, kw, qo, ko, 32, 16)
    bad = list(qkv)
    bad[1] = torch.zeros(2, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.qk_norm_sharded(bad, qw, kw, qo, ko, 32, 16)
    with pytest.raises(ValueError, match="q_weight"):
        B.qk_norm_sharded(qkv, qw[:16], kw, qo, ko, 32, 16)
    with pytest.raises(ValueError, match="k_weight"):
        B.qk_norm_sharded(qkv, qw, torch.ones(8, dtype=torch.bfloat16), qo, ko, 32, 16)
    with pytest.raises(TypeError, match="dtype"):
        B.qk_norm_sharded(qkv, qw, kw.half(), qo, ko, 32, 16)
    with pytest.raises(ValueError):
        B.qk_norm_sharded(qkv, qw, kw, qo[:1], ko, 32, 16)
    with pytest.raises(ValueError, match="multiples"):
        B.qk_norm_sharded(qkv, qw, kw, qo, ko, 31, 16)
    short = [torch.empty(2, 16, dtype=torch.bfloat16) for _ in range(2)]
    with pytest.raises(ValueError, match="dense"):
        B.qk_norm_sharded(qkv, qw, kw, short, ko, 32, 16)
