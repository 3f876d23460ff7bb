"""The parity checker itself, on hand-made values (CPU only).

A checker that is looser than the stated tolerance would let every GPU test
pass a kernel that is off by one unit in the last place of bf16 (up to about
1.2e-2 relative).  These cases pin it: per element |g - o| <= 4e-3 |o|, and
the one-ulp clause only where o is zero or below the format's smallest
normal number."""
import numpy as np
import pytest

import parity as P


def bf16_bits(x):
    import torch
    return np.array([torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()
                     ], dtype=np.int16).view(np.uint16)


def fp16_bits(x):
    return np.array([x], dtype=np.float16).view(np.uint16)


def test_bf16_one_ulp_off_normal_fails():
    # o = 1 + 2^-9 rounds to 1.0; the neighbour 1 + 2^-7 is 5.8e-3 away
    o = np.array([1.0 + 2.0 ** -9])
    assert P.check_y(np.array([0x3F80], dtype=np.uint16), o, "bf16")["ulp_clause"] == 0
    with pytest.raises(AssertionError):
        P.check_y(np.array([0x3F81], dtype=np.uint16), o, "bf16")


def test_bf16_near_midpoint_within_relative_bound_passes():
    # just above the midpoint 1 + 2^-8: RNE is 1 + 2^-7, but 1.0 is within
    # 3.91e-3 relative (a double rounding at a midpoint stays inside 4e-3)
    o = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30])
    st = P.check_y(np.array([0x3F80], dtype=np.uint16), o, "bf16")
    assert st["ulp_clause"] == 0 and st["max_rel"] < 4e-3


def test_bf16_tiny_normal_has_no_ulp_clause():
    o = np.array([1e-30])
    good = bf16_bits(1e-30)
    P.check_y(good, o, "bf16")
    with pytest.raises(AssertionError):
        P.check_y(good + np.uint16(1), o, "bf16")


def test_fp16_subnormal_one_ulp_passes_two_fail():
    u = 2.0 ** -24                      # fp16 subnormal spacing
    o = np.array([3.3 * u])             # RNE = 3u (9% off); 4u is 21% off, one unit away
    st = P.check_y(fp16_bits(3 * u), o, "fp16")
    assert st["ulp_clause"] == 1 and st["tiny"] == 1
    st = P.check_y(fp16_bits(4 * u), o, "fp16")
    assert st["ulp_clause"] == 1
    with pytest.raises(AssertionError):
        P.check_y(fp16_bits(5 * u), o, "fp16")


def test_zero_output():
    o = np.array([0.0])
    P.check_y(np.array([0x0000], dtype=np.uint16), o, "bf16")
    P.check_y(np.array([0x8000], dtype=np.uint16), o, "bf16")      # -0
    assert P.check_y(np.array([0x0001], dtype=np.uint16), o, "fp16")["ulp_clause"] == 1
    with pytest.raises(AssertionError):
        P.check_y(np.array([0x0002], dtype=np.uint16), o, "fp16")


def test_fp16_normal_relative_bound():
    # fp16 half-unit is 2^-11 relative: a value 3e-3 off passes, 5e-3 fails
    o = np.array([1.0])
    P.check_y(fp16_bits(1.0 + 3e-3), o, "fp16")
    with pytest.raises(AssertionError):
        P.check_y(fp16_bits(1.0 + 5e-3), o, "fp16")
