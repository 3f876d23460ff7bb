"""Pins for the fp64 CPU oracle: each function is tied to something other
than itself -- a library routine in a special case, exact rational
arithmetic, closed forms derived by hand, invariances the definitions imply,
and exhaustive comparisons of the number-format code with torch's CPU casts.

A plausible slip in the oracle (a dropped residual or partial, a wrong
denominator, eps outside the root, a missing Gemma bias, a wrong shard
slice, a transposed operand, a wrong rounding tie) fails at least one test
here; ``test_mutations_are_caught`` plants such slips in copies of the oracle
source and checks that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import exact
from tensor_allreduce_residual_ar_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
U = 2.0 ** -53


def _to_bits(values, dtype):
    t = torch.tensor(values, dtype=torch.float64).to(torch.float32)
    td = t.to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    assert torch.equal(td.to(torch.float32), t), "fixture value not exact in dtype"
    return wl.bits(td)


def _expr(s):
    return eval(s, {"__builtins__": {}, "sqrt": math.sqrt})


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dt,td", [(oracle.BF16, torch.bfloat16), (oracle.FP16, torch.float16)])
def test_decode16_exhaustive_vs_torch(dt, td):
    codes = np.arange(65536, dtype=np.uint16)
    ours = oracle.decode16(codes, dt)
    ref = torch.from_numpy(codes.view(np.int16)).view(td).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


@pytest.mark.parametrize("dt,td", [(oracle.BF16, torch.bfloat16), (oracle.FP16, torch.float16)])
def test_round16_midpoints_vs_torch(dt, td):
    """Every midpoint between neighbouring finite values (ties to even), the
    midpoints nudged by one fp32 ulp either way, and the values themselves,
    against torch's fp32 -> 16-bit cast (all test values are fp32-exact)."""
    codes = np.arange(0, 0x7F80 if dt == oracle.BF16 else 0x7C00, dtype=np.uint16)
    vals = oracle.decode16(codes, dt)
    mids = (vals[:-1] + vals[1:]) / 2.0
    f32 = mids.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), mids)
    up = np.nextafter(f32, np.float32(np.inf))
    dn = np.nextafter(f32, np.float32(-np.inf))
    xs = np.concatenate([vals, mids, up, dn, -mids, -vals]).astype(np.float32)
    ref = wl.bits(torch.from_numpy(xs).to(td))
    ours = oracle.round16(xs.astype(np.float64), dt)
    assert np.array_equal(ours, ref)


def test_round16_fp16_random_doubles_vs_numpy():
    """numpy rounds float64 -> float16 directly (one rounding)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal(200000) * np.exp2(rng.integers(-30, 17, 200000))
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.round16(x, oracle.FP16), ref)


def test_round16_overflow_and_specials():
    x = np.array([np.inf, -np.inf, 65520.0, 65519.99, 3.3962e38, 0.0, -0.0, 3.3961e38])
    fp = oracle.round16(x, oracle.FP16)
    assert list(fp[:4]) == [0x7C00, 0xFC00, 0x7C00, 0x7BFF]
    assert list(fp[5:7]) == [0x0000, 0x8000]
    bf = oracle.round16(x, oracle.BF16)
    assert bf[0] == 0x7F80 and bf[4] == 0x7F80 and bf[7] == 0x7F7F
    assert oracle.round16(np.array([np.nan]), oracle.BF16)[0] & 0x7FFF > 0x7F80


def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_encode_roundtrip_midpoints_vs_torch():
    codes = np.arange(0, 0x7F, dtype=np.uint8)     # all finite non-negative codes
    vals = oracle.e4m3_decode(codes)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)
    assert np.array_equal(oracle.e4m3_encode(-vals)[1:], codes[1:] | 0x80)
    mids = (vals[:-1] + vals[1:]) / 2.0
    f32 = mids.astype(np.float32)
    up = np.nextafter(f32, np.float32(np.inf))
    dn = np.nextafter(f32, np.float32(-np.inf))
    xs = np.concatenate([mids, up, dn, -mids, -up]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(xs.astype(np.float64))
    assert np.array_equal(ours, ref)
    # ties go to the even code: e.g. 1 + 1/16 sits between 0x38 and 0x39
    assert oracle.e4m3_encode(np.array([1.0625]))[0] == 0x38
    assert oracle.e4m3_encode(np.array([1.1875]))[0] == 0x3A


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e30, np.inf, -1e30, -np.inf])
    assert list(oracle.e4m3_encode(x)) == [0x7E] * 6 + [0xFE] * 2
    assert oracle.e4m3_encode(np.array([np.nan]))[0] == 0x7F


# ----------------------------------------------------------------------------
# RMSNorm family
# ----------------------------------------------------------------------------

def _norm(inp, gemma=None, want_r=True, want_inv=False, residual=True):
    dt = wl.DTYPE_CODE[inp.dtype]
    return oracle.ar_add_rmsnorm([wl.bits(p) for p in inp.partials],
                                 wl.bits(inp.residual) if (inp.residual is not None and residual) else None,
                                 wl.bits(inp.weight), inp.eps,
                                 inp.gemma if gemma is None else gemma, dt,
                                 want_r=want_r, want_inv=want_inv)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("gemma", [False, True])
def test_w1_zero_residual_is_torch_rms_norm(dtype, gemma):
    """W = 1 and no residual: plain RMSNorm, torch's rms_norm in fp64."""
    inp = wl.make_norm_inputs(wl.DECODE, 8, dtype, W=1, H=1024, residual=False, seed=7)
    got = _norm(inp, gemma=gemma)["y"]
    x = inp.partials[0].to(torch.float64)
    w = inp.weight.to(torch.float64)
    ref = torch.nn.functional.rms_norm(x, (1024,), (1.0 + w) if gemma else w, eps=inp.eps)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-13, atol=1e-300)
    # a zero residual tensor is the same as no residual
    zero = torch.zeros_like(inp.partials[0])
    got0 = oracle.ar_add_rmsnorm([wl.bits(inp.partials[0])], wl.bits(zero), wl.bits(inp.weight),
                                 inp.eps, gemma, wl.DTYPE_CODE[dtype])["y"]
    assert np.array_equal(got0, got)


def test_residual_counts_like_a_partial():
    """residual + sum of W partials == sum of W+1 partials, no residual."""
    inp = wl.make_norm_inputs(wl.TINY, 4, seed=11, H=512)
    a = _norm(inp)
    b = oracle.ar_add_rmsnorm([wl.bits(p) for p in [inp.residual] + inp.partials], None,
                              wl.bits(inp.weight), inp.eps, False, 0)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["r"], b["r"])


def test_permutation_invariance():
    inp = wl.make_norm_inputs(wl.PREFILL, 6, seed=3, H=1024)
    base = _norm(inp)
    rng = np.random.default_rng(0)
    for _ in range(3):
        perm = rng.permutation(inp.W)
        got = oracle.ar_add_rmsnorm([wl.bits(inp.partials[i]) for i in perm], wl.bits(inp.residual),
                                    wl.bits(inp.weight), inp.eps, False, 0)
        assert np.array_equal(got["y"], base["y"]) and np.array_equal(got["r"], base["r"])


def test_scale_invariance():
    """Scaling every activation by 2^k and eps by 4^k leaves y unchanged and
    scales r by 2^k (power-of-two scaling is exact)."""
    inp = wl.make_norm_inputs(wl.TINY, 4, seed=5, H=256)
    base = _norm(inp)
    for k in (-3, 4):
        s = 2.0 ** k
        parts = [wl.bits((p.float() * s).to(torch.bfloat16)) for p in inp.partials]
        res = wl.bits((inp.residual.float() * s).to(torch.bfloat16))
        got = oracle.ar_add_rmsnorm(parts, res, wl.bits(inp.weight), inp.eps * 4.0 ** k, False, 0)
        assert np.array_equal(got["y"], base["y"])
        assert np.array_equal(got["r"], base["r"] * s)


@pytest.mark.parametrize("gemma", [False, True])
def test_row_rms_identity(gemma):
    """mean_h (y_h / w_eff_h)^2 == ms / (ms + eps) for every row."""
    inp = wl.make_norm_inputs(wl.DECODE, 5, "bf16", H=2048, seed=9)
    inp.eps = 0.05   # large enough that the identity differs visibly from 1
    out = _norm(inp, gemma=gemma)
    w = inp.weight.double().numpy()
    weff = 1.0 + w if gemma else w
    ms = (out["r"] ** 2).mean(axis=1)
    lhs = ((out["y"] / weff) ** 2).mean(axis=1)
    np.testing.assert_allclose(lhs, ms / (ms + inp.eps), rtol=1e-13)


def _exact_compare(inp, gemma, bound_scale=1.0):
    decode = exact.bf16 if inp.dtype == "bf16" else exact.fp16
    parts = [wl.bits(p).tolist() for p in inp.partials]
    res = wl.bits(inp.residual).tolist() if inp.residual is not None else None
    r_x, y_x = exact.rmsnorm_rows(parts, res, wl.bits(inp.weight).tolist(),
                                  exact.Fraction(inp.eps), gemma, decode)
    out = _norm(inp, gemma=gemma)
    H = inp.H
    # the oracle's only roundings: a sequential fp64 sum of H positive squares
    # ((H-1) u), the mean, eps, sqrt, one division, one product.
    tol = (H / 2.0 + 4.0) * U * bound_scale
    for t in range(inp.T):
        for h in range(H):
            assert out["r"][t, h] == float(r_x[t][h])      # the sum is exact
            ye = float(y_x[t][h])
            assert abs(out["y"][t, h] - ye) <= tol * abs(ye) + 1e-300, (t, h)


@pytest.mark.parametrize("dtype,gemma,res", [("bf16", False, True), ("fp16", True, True),
                                             ("bf16", True, False), ("fp16", False, False)])
def test_exact_rational_2x8(dtype, gemma, res):
    for seed in range(4):
        inp = wl.make_norm_inputs(wl.DECODE, 2, dtype, H=8, W=3, residual=res, seed=100 + seed)
        _exact_compare(inp, gemma)


def test_exact_rational_tiny_config():
    """The whole tiny workload (T=16, H=4096, W=2) in exact arithmetic."""
    inp = wl.make_norm_inputs(wl.TINY, 16)
    _exact_compare(inp, False)


def test_closed_forms():
    with open(GOLDEN) as f:
        gold = json.load(f)
    for case in gold["norm_cases"]:
        dt = case["dtype"]
        parts = [_to_bits(p, dt) for p in case["partials"]]
        parts = [p.reshape(1, -1) for p in parts]
        res = _to_bits(case["residual"], dt).reshape(1, -1) if case["residual"] is not None else None
        out = oracle.ar_add_rmsnorm(parts, res, _to_bits(case["weight"], dt), case["eps"],
                                    case["gemma"], wl.DTYPE_CODE[dt])
        r_ref = np.array([_expr(s) for s in case["r"]])
        y_ref = np.array([_expr(s) for s in case["y"]])
        assert np.array_equal(out["r"][0], r_ref), case["name"]
        np.testing.assert_allclose(out["y"][0], y_ref, rtol=4 * U, atol=0, err_msg=case["name"])


# ----------------------------------------------------------------------------
# FP8 per-group output
# ----------------------------------------------------------------------------

def test_fp8_closed_forms():
    with open(GOLDEN) as f:
        gold = json.load(f)
    for case in gold["fp8_cases"]:
        H = case["H"]
        row = np.zeros(H)
        row[:len(case["partial_head"])] = case["partial_head"]
        part = _to_bits(row, case["dtype"]).reshape(1, H)
        wt = _to_bits(np.full(H, case["weight_value"], dtype=np.float64), case["dtype"])
        y = oracle.ar_add_rmsnorm([part], None, wt, case["eps"], case["gemma"], 0)["y"]
        q, s64, s32 = oracle.quant_fp8_group(y, case["group"])
        np.testing.assert_allclose(s64[0], [_expr(s) for s in case["scales"]], rtol=4 * U, atol=0)
        head = [int(c, 16) for c in case["codes_head"]]
        assert list(q[0, :len(head)]) == head, case["name"]
        assert np.all(q[0, len(head):] == int(case["codes_tail"], 16))


def _ordinal(codes):
    c = codes.astype(np.int32)
    return np.where(c & 0x80, -(c & 0x7F), c)


def test_fp8_group_invariants():
    inp = wl.make_norm_inputs(wl.FP8, 8)
    y = _norm(inp)["y"]
    q, s64, s32 = oracle.quant_fp8_group(y, 128)
    T, H = y.shape
    G = H // 128
    mag = q & 0x7F
    # every non-zero group reaches the largest finite code (448) exactly once or more
    assert np.all(mag.reshape(T, G, 128).max(axis=2) == 0x7E)
    # scale is amax/448 in fp64, and its fp32 twin is within one fp32 rounding
    amax = np.abs(y).reshape(T, G, 128).max(axis=2)
    assert np.array_equal(s64, amax / 448.0)
    np.testing.assert_allclose(s32, s64, rtol=2 ** -22)
    # dequantised value within half an e4m3 step of y (plus fp32 slack)
    deq = oracle.e4m3_decode(q) * np.repeat(s64, 128, axis=1)
    vals = np.abs(oracle.e4m3_decode(mag))
    nxt = np.abs(oracle.e4m3_decode(np.minimum(mag + 1, 0x7E)))
    prv = np.abs(oracle.e4m3_decode(np.maximum(mag.astype(np.int32) - 1, 0).astype(np.uint8)))
    step = np.maximum(nxt - vals, vals - prv) * np.repeat(s64, 128, axis=1)
    assert np.all(np.abs(deq - y) <= 0.5 * step + 1e-6 * np.abs(y) + 1e-300)
    # signs agree wherever the code is non-zero
    nz = mag != 0
    assert np.array_equal(np.signbit(y[nz]), (q[nz] & 0x80) != 0)


def test_fp8_zero_group():
    y = np.zeros((2, 256))
    y[1, :128] = np.linspace(-3, 3, 128)
    q, s64, s32 = oracle.quant_fp8_group(y, 128)
    assert np.all(q[0] == 0) and np.all(s64[0] == 0) and np.all(q[1, 128:] == 0)
    assert s64[1, 0] == 3.0 / 448.0


# ----------------------------------------------------------------------------
# sharded QK-norm
# ----------------------------------------------------------------------------

def test_qk_equals_torch_rms_norm_of_concatenation():
    inp = wl.make_qk_inputs(wl.QK, 3, seed=21)
    q_out, k_out = oracle.qk_norm_sharded([wl.bits(x) for x in inp.qkv], wl.bits(inp.q_weight),
                                          wl.bits(inp.k_weight), inp.q_size, inp.kv_size,
                                          inp.eps, 0)
    W, qs, ks = inp.W, inp.q_size // inp.W, inp.kv_size // inp.W
    Q = torch.cat([x[:, :qs] for x in inp.qkv], dim=1).double()
    K = torch.cat([x[:, qs:qs + ks] for x in inp.qkv], dim=1).double()
    Qn = torch.nn.functional.rms_norm(Q, (inp.q_size,), inp.q_weight.double(), eps=inp.eps)
    Kn = torch.nn.functional.rms_norm(K, (inp.kv_size,), inp.k_weight.double(), eps=inp.eps)
    for w in range(W):
        np.testing.assert_allclose(q_out[w], Qn[:, w * qs:(w + 1) * qs].numpy(), rtol=1e-13)
        np.testing.assert_allclose(k_out[w], Kn[:, w * ks:(w + 1) * ks].numpy(), rtol=1e-13)


def test_qk_single_shard_is_plain_rmsnorm():
    inp = wl.make_qk_inputs(wl.QK, 2, W=1, q_size=64, kv_size=32, seed=4)
    q_out, k_out = oracle.qk_norm_sharded([wl.bits(inp.qkv[0])], wl.bits(inp.q_weight),
                                          wl.bits(inp.k_weight), 64, 32, inp.eps, 0)
    q_only = inp.qkv[0][:, :64].contiguous()
    ref = oracle.ar_add_rmsnorm([wl.bits(q_only)], None, wl.bits(inp.q_weight), inp.eps, False, 0)["y"]
    np.testing.assert_allclose(q_out[0], ref, rtol=1e-15)


def test_qk_exact_rational():
    inp = wl.make_qk_inputs(wl.QK, 2, W=4, q_size=32, kv_size=16, seed=8)
    shards = [wl.bits(x).tolist() for x in inp.qkv]
    qx, kx = exact.qk_rows(shards, wl.bits(inp.q_weight).tolist(), wl.bits(inp.k_weight).tolist(),
                           32, 16, exact.Fraction(inp.eps), exact.bf16)
    q_out, k_out = oracle.qk_norm_sharded([wl.bits(x) for x in inp.qkv], wl.bits(inp.q_weight),
                                          wl.bits(inp.k_weight), 32, 16, inp.eps, 0)
    for w in range(4):
        for t in range(2):
            np.testing.assert_allclose(q_out[w, t], [float(v) for v in qx[w][t]], rtol=24 * U)
            np.testing.assert_allclose(k_out[w, t], [float(v) for v in kx[w][t]], rtol=16 * U)


def test_qk_closed_forms():
    with open(GOLDEN) as f:
        gold = json.load(f)
    for case in gold["qk_cases"]:
        shards = [_to_bits(s, case["dtype"]).reshape(1, -1) for s in case["shards"]]
        q_out, k_out = oracle.qk_norm_sharded(shards, _to_bits(case["q_weight"], case["dtype"]),
                                              _to_bits(case["k_weight"], case["dtype"]),
                                              case["q_size"], case["kv_size"], case["eps"], 0)
        for w in range(len(shards)):
            np.testing.assert_allclose(q_out[w, 0], [_expr(s) for s in case["q_out"][w]], rtol=4 * U)
            np.testing.assert_allclose(k_out[w, 0], [_expr(s) for s in case["k_out"][w]], rtol=4 * U)


# ----------------------------------------------------------------------------
# mutation check: plausible slips planted in copies of the oracle are caught
# ----------------------------------------------------------------------------

MUTATIONS = {
    "drop_residual": ("double r = residual ? oracle_decode16(residual[t * H + h], dtype) : 0.0;",
                      "double r = 0.0;"),
    "drop_last_partial": ("for (int w = 0; w < W; ++w)\n                r +=",
                          "for (int w = 0; w < W - 1; ++w)\n                r +="),
    "mean_over_H_minus_1": ("double ms = sumsq / (double)H;", "double ms = sumsq / (double)(H - 1);"),
    "eps_outside_root": ("double denom = sqrt(ms + eps);", "double denom = sqrt(ms) + eps;"),
    "no_gemma_bias": ("double weff = gemma ? 1.0 + wv : wv;", "double weff = wv;"),
    "weight_reversed": ("oracle_decode16(weight[h], dtype)", "oracle_decode16(weight[H - 1 - h], dtype)"),
    "qk_weight_slice": ("oracle_decode16(q_weight[w * qs + j], dtype)", "oracle_decode16(q_weight[j], dtype)"),
    "qk_denominators_swapped": ("ssq_q / (double)q_size", "ssq_q / (double)kv_size"),
    "qk_k_uses_q_rms": ("oracle_decode16(x[qs + j], dtype) / den_k", "oracle_decode16(x[qs + j], dtype) / den_q"),
    "round16_ties_up": ("if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))\n        n = fl + 1.0;\n    /* value",
                        "if (rem >= 0.5)\n        n = fl + 1.0;\n    /* value"),
    "e4m3_ties_up": ("if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))\n        n = fl + 1.0;\n    double val = ldexp(n, q_exp);\n    if (val >= 448.0)",
                     "if (rem >= 0.5)\n        n = fl + 1.0;\n    double val = ldexp(n, q_exp);\n    if (val >= 448.0)"),
    "fp8_max_240": ("volatile float s32 = amax32 / 448.0f;", "volatile float s32 = amax32 / 240.0f;"),
    "e4m3_bias_8": ("mag = ldexp((double)(8u | frac), (int)exp - 7 - 3);",
                    "mag = ldexp((double)(8u | frac), (int)exp - 8 - 3);"),
    "bf16_fraction_bits": ("bits & 0x7Fu, 8, 7", "bits & 0x3Fu, 8, 7"),
    "fp16_subnormal_scale": ("mag = ldexp((double)frac, 1 - bias - frac_bits);",
                             "mag = ldexp((double)frac, -bias - frac_bits);"),
}


def _pin_checks():
    """The quick pins, as plain calls; returns the names that failed."""
    checks = [
        ("torch_rms_norm_bf16", lambda: test_w1_zero_residual_is_torch_rms_norm("bf16", False)),
        ("torch_rms_norm_gemma", lambda: test_w1_zero_residual_is_torch_rms_norm("fp16", True)),
        ("exact_2x8", lambda: [test_exact_rational_2x8(*a) for a in
                               [("bf16", False, True), ("fp16", True, True)]]),
        ("closed_forms", test_closed_forms),
        ("fp8_closed_forms", test_fp8_closed_forms),
        ("fp8_invariants", test_fp8_group_invariants),
        ("qk_torch", test_qk_equals_torch_rms_norm_of_concatenation),
        ("qk_closed_forms", test_qk_closed_forms),
        ("round16_bf16", lambda: test_round16_midpoints_vs_torch(oracle.BF16, torch.bfloat16)),
        ("round16_fp16", lambda: test_round16_midpoints_vs_torch(oracle.FP16, torch.float16)),
        ("decode16_fp16", lambda: test_decode16_exhaustive_vs_torch(oracle.FP16, torch.float16)),
        ("e4m3", test_e4m3_encode_roundtrip_midpoints_vs_torch),
        ("e4m3_decode", test_e4m3_decode_exhaustive_vs_torch),
    ]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


def test_mutations_are_caught(tmp_path):
    assert _pin_checks() == []        # the real oracle passes every quick pin
    src = oracle.source_text()
    for name, (old, new) in MUTATIONS.items():
        assert src.count(old) >= 1, f"mutation {name} does not apply"
        path = oracle.compile_variant(src.replace(old, new), str(tmp_path / f"m_{name}.so"))
        with oracle.use_library(path):
            failed = _pin_checks()
        assert failed, f"planted slip '{name}' was not caught by any pin"
