"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every entry point ``include/*.h`` declares, rejects bad
arguments with the documented status before touching the device, treats
T == 0 as a no-op, and loads / rejects plan tables as documented."""
import ctypes
import glob
import json
import os
import re

import pytest

from tensor_allreduce_residual_ar_b200 import build as arbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, EINVAL, EALIGN, EUNSUP = 0, 1, 2, 3


@pytest.fixture(scope="module")
def clib():
    path = arbuild.build()
    lib = ctypes.CDLL(path)
    P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    PP = ctypes.POINTER(ctypes.c_void_p)
    lib.ar_add_rmsnorm.argtypes = [PP, P, P, P, P, i64, i64, i32, f32, i32, i32, P]
    lib.ar_add_rmsnorm_quant_fp8_group.argtypes = [PP, P, P, P, P, P, P, i64, i64, i32, i32, f32,
                                                   i32, i32, P]
    lib.ar_add_rmsnorm_quant_fp8_group_strided.argtypes = [PP, P, P, P, P, i64, i64, P, P, i64, i64,
                                                           i32, i32, f32, i32, i32, P]
    lib.qk_norm_sharded.argtypes = [PP, P, P, PP, PP, i64, i64, i64, i32, f32, i32, P]
    lib.ar_plan_query.argtypes = [i32, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_int)]
    lib.ar_plan_load.argtypes = [ctypes.c_char_p]
    lib.ar_plan_force.argtypes = [i32, i32]
    lib.ar_status_string.restype = ctypes.c_char_p
    yield lib
    lib.ar_plan_load(None)
    for v in range(3):
        lib.ar_plan_force(v, 0)


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = "\n".join(l for l in open(h).read().splitlines() if not l.lstrip().startswith("#"))
        names |= set(re.findall(r"AR_API\s+[\w\s\*]*?\b(\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(clib):
    names = _declared_symbols()
    assert {"ar_add_rmsnorm", "ar_add_rmsnorm_quant_fp8_group", "qk_norm_sharded",
            "ar_plan_query", "ar_status_string"} <= names
    for n in names:
        assert hasattr(clib, n), n


def test_library_has_no_oracle_dependency():
    """The product library links nothing from the oracle."""
    for src in arbuild.sources() + glob.glob(os.path.join(ROOT, "tensor_allreduce_residual_ar_b200", "*.py")):
        text = open(src).read()
        assert "oracle" not in re.sub(r"#.*|//.*", "", text).lower() or src.endswith("workloads.py"), src


def _ptrs(*vals):
    return (ctypes.c_void_p * len(vals))(*vals)


A = 0x100000          # fake, 16-byte aligned device addresses: never dereferenced
B, C_, D, E = A + 0x1000, A + 0x2000, A + 0x3000, A + 0x4000


def test_norm_argument_errors(clib):
    parts = _ptrs(A, B)
    f = clib.ar_add_rmsnorm
    assert f(None, None, C_, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EINVAL
    assert f(parts, None, None, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EINVAL      # weight
    assert f(parts, None, C_, None, None, 4, 64, 2, 1e-6, 0, 0, None) == EINVAL     # out
    assert f(parts, None, C_, D, None, 4, 60, 2, 1e-6, 0, 0, None) == EINVAL        # H % 8
    assert f(parts, None, C_, D, None, 4, 0, 2, 1e-6, 0, 0, None) == EINVAL
    assert f(parts, None, C_, D, None, -1, 64, 2, 1e-6, 0, 0, None) == EINVAL
    assert f(parts, None, C_, D, None, 4, 64, 0, 1e-6, 0, 0, None) == EINVAL        # W
    assert f(_ptrs(*([A] * 17)), None, C_, D, None, 4, 64, 17, 1e-6, 0, 0, None) == EINVAL
    assert f(parts, None, C_, D, None, 4, 64, 2, 1e-6, 0, 2, None) == EINVAL        # dtype
    assert f(parts, None, C_, D, None, 4, 64, 2, -1.0, 0, 0, None) == EINVAL        # eps
    assert f(parts, None, C_, D, None, 4, 64, 2, float("nan"), 0, 0, None) == EINVAL
    assert f(_ptrs(A, None), None, C_, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EINVAL
    assert f(_ptrs(A, B + 2), None, C_, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EALIGN
    assert f(parts, E + 8, C_, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EALIGN       # residual
    assert f(parts, None, C_ + 4, D, None, 4, 64, 2, 1e-6, 0, 0, None) == EALIGN    # weight
    assert f(parts, None, C_, D + 2, None, 4, 64, 2, 1e-6, 0, 0, None) == EALIGN    # out
    assert f(parts, None, C_, D, E + 6, 4, 64, 2, 1e-6, 0, 0, None) == EALIGN       # res out
    assert f(parts, None, C_, D, None, 4, 65536 + 8, 2, 1e-6, 0, 0, None) == EUNSUP
    # T == 0: valid, nothing launched (no device needed)
    assert f(parts, E, C_, D, E, 0, 64, 2, 1e-6, 1, 1, None) == OK


def test_fp8_argument_errors(clib):
    parts = _ptrs(A, B)
    f = clib.ar_add_rmsnorm_quant_fp8_group
    args = lambda **kw: dict(dict(q=D, s=E, y=None, ro=None, T=4, H=256, W=2, g=128), **kw)
    def call(**kw):
        a = args(**kw)
        return f(parts, None, C_, a["q"], a["s"], a["y"], a["ro"], a["T"], a["H"], a["W"], a["g"],
                 1e-6, 0, 0, None)
    assert call(q=None) == EINVAL
    assert call(s=None) == EINVAL
    assert call(g=64) == EINVAL
    assert call(H=200) == EINVAL            # H not a multiple of the group
    assert call(q=D + 8) == EALIGN
    assert call(s=E + 2) == EALIGN
    assert call(y=A + 4) == EALIGN
    assert call(s=E + 4, T=0) == OK         # scales need only 4-byte alignment


def test_fp8_scale_strides(clib):
    """Scale layouts: every (row, group) needs its own slot; checked before
    any device access."""
    parts = _ptrs(A, B)
    f = clib.ar_add_rmsnorm_quant_fp8_group_strided
    def call(st, sg, T=5, H=256):              # G = 2 groups
        return f(parts, None, C_, D, E, st, sg, None, None, T, H, 2, 128, 1e-6, 0, 0, None)
    assert call(1, 1) == EINVAL                # rows overlap groups
    assert call(-2, 1) == EINVAL
    assert call(2, 0) == EINVAL
    assert call(1, 4) == EINVAL                # column-major needs stride_g >= T
    assert call(0, 1) == EINVAL
    assert call(2, 1, T=0) == OK               # row-major
    assert call(1, 5, T=0) == OK               # transposed [G, T]
    assert call(0, 1, T=0) == OK               # no rows: the row stride is free
    assert call(3, 0, T=0, H=128) == OK        # one group: the group stride is free


def test_qk_argument_errors(clib):
    f = clib.qk_norm_sharded
    qkv, qo, ko = _ptrs(A, B), _ptrs(C_, D), _ptrs(E, E + 0x1000)
    base = dict(T=3, q=64, kv=32, W=2)
    def call(qkv=qkv, qo=qo, ko=ko, **kw):
        a = dict(base, **kw)
        return f(qkv, A, B, qo, ko, a["T"], a["q"], a["kv"], a["W"], 1e-6, 0, None)
    assert call(q=63) == EINVAL             # not a multiple of W
    assert call(q=48, kv=16, W=4) == EINVAL   # kv/W = 4 not a multiple of 8
    assert call(kv=0) == EINVAL
    assert call(W=0) == EINVAL
    assert call(qkv=_ptrs(A, None)) == EINVAL
    assert call(qo=_ptrs(C_, D + 2)) == EALIGN
    assert call(T=0) == OK


def test_withhold_hook_validates(clib):
    clib.ar_test_withhold_row.argtypes = [ctypes.c_int64]
    assert clib.ar_test_withhold_row(-2) == EINVAL
    assert clib.ar_test_withhold_row(-1) == OK


def test_status_strings(clib):
    for s in range(6):
        assert clib.ar_status_string(s).decode().startswith("AR_")
    assert b"unknown" in clib.ar_status_string(99)


def test_plan_table_load_and_reject(clib, tmp_path):
    q = ctypes.c_int(-1)
    clib.ar_plan_load(None)
    assert clib.ar_plan_table_size() == 0
    assert clib.ar_plan_query(0, 8192, 4096, 8, 0, ctypes.byref(q)) == OK
    builtin = q.value
    good = {"entries": [{"variant": 0, "dtype": 0, "W": 8, "H": 4096, "t_lo": 1, "t_hi": 100000,
                         "plan": 3}]}
    p = tmp_path / "good.json"
    p.write_text(json.dumps(good))
    assert clib.ar_plan_load(str(p).encode()) == OK
    assert clib.ar_plan_table_size() == 1
    assert clib.ar_plan_query(0, 8192, 4096, 8, 0, ctypes.byref(q)) == OK and q.value == 3
    # other shapes still take the built-in rule
    assert clib.ar_plan_query(0, 8192, 4096, 8, 1, ctypes.byref(q)) == OK and q.value == builtin
    # corrupt or invalid tables are rejected and the loaded one stays
    bad_texts = [
        "{not json",
        json.dumps({"entries": [{"variant": 0, "dtype": 0, "W": 8, "H": 4096, "t_lo": 1,
                                 "t_hi": 9, "plan": 11}]}),          # QK plan for norm
        json.dumps({"entries": [{"variant": 0, "dtype": 0, "W": 8, "H": 4096, "t_lo": 9,
                                 "t_hi": 1, "plan": 1}]}),           # empty range
        json.dumps({"entries": [{"variant": 0, "dtype": 0, "W": 8, "H": 4096, "t_lo": 1,
                                 "t_hi": 9, "plna": 1}]}),           # typo
        json.dumps({"entries": [{"variant": 0, "dtype": 0, "W": 8, "H": 4096, "t_lo": 1,
                                 "t_hi": 9, "plan": 1.5}]}),         # not an integer
        json.dumps({"entries": []}) + " trailing",
    ]
    for i, text in enumerate(bad_texts):
        bp = tmp_path / f"bad{i}.json"
        bp.write_text(text)
        assert clib.ar_plan_load(str(bp).encode()) == EINVAL, text
        assert clib.ar_plan_table_size() == 1
    assert clib.ar_plan_load(str(tmp_path / "missing.json").encode()) == EINVAL
    assert clib.ar_plan_load(None) == OK and clib.ar_plan_table_size() == 0


def test_qk_inplace_form_must_cover_every_shard(clib):
    """In-place QK (q_out[w] == qkv[w], k_out[w] == qkv[w] + qs) is all or
    nothing; a mixture is an argument error, found before any device access."""
    W, qs, ks = 2, 64, 32
    base = [0x100000, 0x200000]
    qkv = _ptrs(*base)
    inplace_q = _ptrs(*base)
    inplace_k = _ptrs(*[b + 2 * qs for b in base])
    dense_q = _ptrs(0x300000, 0x400000)
    dense_k = _ptrs(0x500000, 0x600000)
    f = clib.qk_norm_sharded
    # T = 0: validated, nothing launched
    assert f(qkv, C_, D, inplace_q, inplace_k, 0, W * qs, W * ks, W, 1e-6, 0, None) == OK
    assert f(qkv, C_, D, dense_q, dense_k, 0, W * qs, W * ks, W, 1e-6, 0, None) == OK
    mixed_q = _ptrs(base[0], 0x400000)
    mixed_k = _ptrs(base[0] + 2 * qs, 0x600000)
    assert f(qkv, C_, D, mixed_q, mixed_k, 0, W * qs, W * ks, W, 1e-6, 0, None) == EINVAL
    bad_k = _ptrs(base[0] + 2 * qs + 16, base[1] + 2 * qs)
    assert f(qkv, C_, D, inplace_q, bad_k, 0, W * qs, W * ks, W, 1e-6, 0, None) == EINVAL


def test_plan_force(clib):
    q = ctypes.c_int(-1)
    assert clib.ar_plan_force(0, 11) == EINVAL      # QK plan for the norm variant
    assert clib.ar_plan_force(2, 1) == EINVAL
    assert clib.ar_plan_force(3, 1) == EINVAL
    assert clib.ar_plan_force(0, 10) == OK          # PERSIST_C2_AHEAD, the last norm plan
    assert clib.ar_plan_force(0, 11) == EINVAL
    assert clib.ar_plan_force(2, 8) == EINVAL
    assert clib.ar_plan_force(2, 18) == OK          # QK_RING, the last QK plan
    assert clib.ar_plan_force(2, 19) == EINVAL
    assert clib.ar_plan_force(0, 16) == EINVAL
    assert clib.ar_plan_force(2, 0) == OK
    assert clib.ar_plan_force(0, 0) == OK
    assert clib.ar_plan_force(1, 4) == OK
    assert clib.ar_plan_query(1, 5, 5120, 4, 0, ctypes.byref(q)) == OK and q.value == 4
    assert clib.ar_plan_force(1, 0) == OK
    assert clib.ar_plan_query(2, 1, 7168, 8, 0, ctypes.byref(q)) == OK and 11 <= q.value <= 14


def test_plan_ids_agree_across_header_library_tuner_and_tests(clib):
    """Every plan id the header names is accepted for its variant and
    nothing else is; the tuner and the every-plan GPU tests cover exactly
    those ids."""
    import re
    from tensor_allreduce_residual_ar_b200 import tune
    import test_parity_gpu as tp
    hdr = open(os.path.join(ROOT, "include", "ar_rmsnorm.h")).read()
    ids = {name: int(v) for name, v in re.findall(r"AR_PLAN_(\w+) = (\d+)", hdr)}
    qk = {v for n, v in ids.items() if n.startswith("QK_")}
    norm = {v for n, v in ids.items() if v != 0 and not n.startswith("QK_")}
    for variant, valid in ((0, norm), (1, norm), (2, qk)):
        accepted = {pid for pid in range(1, 40) if clib.ar_plan_force(variant, pid) == OK}
        clib.ar_plan_force(variant, 0)
        assert accepted == valid, (variant, sorted(accepted), sorted(valid))
    assert set(tune.NORM_PLANS) == norm and set(tune.QK_PLANS) == qk
    assert set(tp.NORM_PLANS) == norm and set(tp.QK_PLANS) == qk


def test_builtin_rule_is_capture_static(clib):
    """Same arguments, same plan, however often asked (no state, no data)."""
    q1, q2 = ctypes.c_int(-1), ctypes.c_int(-1)
    clib.ar_plan_load(None)
    for T in (1, 2, 80, 81, 4096, 8192, 32768):
        for v, H in ((0, 8192), (1, 5120), (2, 7168)):
            assert clib.ar_plan_query(v, T, H, 4 if v < 2 else 8, 0, ctypes.byref(q1)) == OK
            assert clib.ar_plan_query(v, T, H, 4 if v < 2 else 8, 0, ctypes.byref(q2)) == OK
            assert q1.value == q2.value


def test_shipped_plan_table_parses(clib):
    path = os.path.join(ROOT, "tensor_allreduce_residual_ar_b200", "plan_table.json")
    if not os.path.exists(path):
        pytest.skip("no plan table shipped yet")
    assert clib.ar_plan_load(path.encode()) == OK
    assert clib.ar_plan_table_size() > 0
    clib.ar_plan_load(None)


def test_tuner_ranges_cover_every_T(clib, tmp_path):
    """The tuner's measured winners become contiguous T ranges that the
    library accepts and that reproduce every winner."""
    from tensor_allreduce_residual_ar_b200.tune import table_from_best
    best = {(0, 0, 4, 8192, 1): 4, (0, 0, 4, 8192, 2): 4, (0, 0, 4, 8192, 16): 3,
            (0, 0, 4, 8192, 80): 2, (1, 0, 4, 5120, 1): 4, (1, 0, 4, 5120, 4096): 5,
            (2, 0, 8, 7168, 1): 14, (2, 0, 8, 7168, 2048): 15}
    table = table_from_best(best)
    assert len(table["entries"]) == 7          # the two T=1,2 plan-4 ranges merged
    p = tmp_path / "t.json"
    p.write_text(json.dumps(table))
    assert clib.ar_plan_load(str(p).encode()) == OK
    q = ctypes.c_int(-1)
    for (v, d, W, H, T), plan in best.items():
        assert clib.ar_plan_query(v, T, H, W, d, ctypes.byref(q)) == OK and q.value == plan
    # between measured points the next measured point's plan applies; beyond
    # the last one the last plan does
    assert clib.ar_plan_query(0, 10, 8192, 4, 0, ctypes.byref(q)) == OK and q.value == 3
    assert clib.ar_plan_query(0, 10**6, 8192, 4, 0, ctypes.byref(q)) == OK and q.value == 2
    clib.ar_plan_load(None)
