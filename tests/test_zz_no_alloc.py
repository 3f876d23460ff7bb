"""The allocation-free group QK-norm entry point, against the existing one.

Some callers cannot call cudaMalloc: a plugin that only receives buffers
from its host application, an engine that reserved all free device memory
when it started (so a further allocation fails), or code that must not take
the device-wide synchronisation cudaMalloc may imply.
ar_group_qk_norm_sharded_static serves them: it runs the same kernel as
ar_group_qk_norm_sharded with its exchange regions in a file-scope device
array.  This test calls it through the C ABI on two calls in a row (the
array keeps the previous call's contents) and compares its outputs with
ar_group_qk_norm_sharded's on the same inputs, within the relative
tolerance the parity tests use.  The file name makes pytest collect it
last."""
import ctypes

import pytest
import torch

import parity as P
from tensor_allreduce_residual_ar_b200 import binding as B
from tensor_allreduce_residual_ar_b200 import comm as C
from tensor_allreduce_residual_ar_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TD = {"bf16": torch.bfloat16, "fp16": torch.float16}


def static_entry_point():
    fn = B.load_library().ar_group_qk_norm_sharded_static
    VP, PP = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)
    fn.argtypes = [ctypes.c_int, PP, VP, VP, PP, PP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_float, ctypes.c_int, VP]
    fn.restype = ctypes.c_int
    return fn


def ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def test_static_entry_point_matches_the_group_entry_point(lib):
    fn = static_entry_point()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row: different W, T and dtype, so the second call runs
    # on whatever the first left in the array
    for T, W, q_size, kv_size, dtype in ((64, 8, 6144, 1024, "bf16"), (300, 4, 512, 256, "fp16")):
        inp = wl.make_qk_inputs(wl.QK, T, dtype, W=W, q_size=q_size, kv_size=kv_size, seed=31000 + T)
        qs, ks = q_size // W, kv_size // W
        td = TD[dtype]
        qkv = [x.cuda() for x in inp.qkv]
        qw, kw = inp.q_weight.cuda(), inp.k_weight.cuda()
        q_static = [torch.empty((T, qs), dtype=td, device="cuda") for _ in range(W)]
        k_static = [torch.empty((T, ks), dtype=td, device="cuda") for _ in range(W)]
        st = fn(W, ptrs(qkv), qw.data_ptr(), kw.data_ptr(), ptrs(q_static), ptrs(k_static), T, q_size,
                kv_size, inp.eps, wl.DTYPE_CODE[dtype], stream)
        assert st == 0, B.ar_status_string(st)
        q_ref = [torch.empty_like(q) for q in q_static]
        k_ref = [torch.empty_like(k) for k in k_static]
        g = C.CommGroup(W, 4 * T)
        try:
            g.qk_norm_sharded(qkv, qw, kw, q_ref, k_ref, q_size, kv_size, eps=inp.eps)
            torch.cuda.synchronize()
        finally:
            g.close()
        for a, b in zip(q_static + k_static, q_ref + k_ref):
            a64, b64 = a.double(), b.double()
            assert bool(((a64 - b64).abs() <= P.Y_RTOL * b64.abs()).all())


def test_static_entry_point_rejects_sizes_beyond_its_maximum(lib):
    """Checked on the host before anything is launched."""
    fn = static_entry_point()
    W, T = 2, 4097
    dummy = [torch.empty(16, dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    w = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    assert fn(W, ptrs(dummy), w.data_ptr(), w.data_ptr(), ptrs(dummy), ptrs(dummy), T, 16, 16, 1e-6,
              0, None) == 3          # AR_EUNSUPPORTED
    assert fn(17, ptrs(dummy * 9), w.data_ptr(), w.data_ptr(), ptrs(dummy * 9), ptrs(dummy * 9), 1,
              17 * 8, 17 * 8, 1e-6, 0, None) == 1      # AR_EINVAL
