"""Exact-rational checker for tiny shapes (Python stdlib only).

TEST INFRASTRUCTURE: pins the fp64 oracle (``oracle.c``) on small inputs.  It
shares no code with the oracle: 16-bit values are decoded here by their own
bit-field arithmetic into ``fractions.Fraction``, sums and squares are exact,
and the one irrational step, the square root, is taken in ``decimal`` at 60
significant digits.

Definitions followed (vLLM PR #54787 report, "关键源码片段": explicit
all_reduce then (Gemma)RMSNorm with residual; vLLM PR #44849 report,
"关键源码片段": MiniMax QK-norm over the full TP width):
    r  = residual + sum_w P_w
    y  = r / sqrt(mean(r^2) + eps) * (w  or  1 + w)
"""
from __future__ import annotations

from decimal import Decimal, getcontext
from fractions import Fraction

getcontext().prec = 60


def frac_from_bits(bits: int, exp_bits: int, frac_bits: int) -> Fraction:
    sign = -1 if (bits >> (exp_bits + frac_bits)) & 1 else 1
    e = (bits >> frac_bits) & ((1 << exp_bits) - 1)
    f = bits & ((1 << frac_bits) - 1)
    bias = (1 << (exp_bits - 1)) - 1
    if e == (1 << exp_bits) - 1:
        raise ValueError("inf/nan has no rational value")
    if e == 0:
        mag = Fraction(f) * Fraction(2) ** (1 - bias - frac_bits)
    else:
        mag = Fraction((1 << frac_bits) + f) * Fraction(2) ** (e - bias - frac_bits)
    return sign * mag


def bf16(bits: int) -> Fraction:
    return frac_from_bits(int(bits), 8, 7)


def fp16(bits: int) -> Fraction:
    return frac_from_bits(int(bits), 5, 10)


def _dec(x: Fraction) -> Decimal:
    return Decimal(x.numerator) / Decimal(x.denominator)


def rmsnorm_rows(partials, residual, weight, eps: Fraction, gemma: bool, decode):
    """partials: list of W lists of rows (lists of 16-bit ints); residual the
    same shape or None; weight a list of 16-bit ints.  Returns (r, y) with r
    exact Fractions and y Decimals (60 digits)."""
    T = len(partials[0])
    H = len(weight)
    w_eff = [(1 + decode(b)) if gemma else decode(b) for b in weight]
    r_rows, y_rows = [], []
    for t in range(T):
        r = []
        for h in range(H):
            acc = decode(residual[t][h]) if residual is not None else Fraction(0)
            for p in partials:
                acc += decode(p[t][h])
            r.append(acc)
        ms = sum((v * v for v in r), Fraction(0)) / H
        denom = _dec(ms + eps).sqrt()
        y_rows.append([_dec(r[h]) / denom * _dec(w_eff[h]) for h in range(H)])
        r_rows.append(r)
    return r_rows, y_rows


def qk_rows(shards, q_weight, k_weight, q_size: int, kv_size: int, eps: Fraction,
            decode):
    """shards: W lists of rows [qs | ks | ks]; returns (q_out, k_out) as
    [W][T][cols] Decimals."""
    W = len(shards)
    T = len(shards[0])
    qs, ks = q_size // W, kv_size // W
    q_out = [[None] * T for _ in range(W)]
    k_out = [[None] * T for _ in range(W)]
    for t in range(T):
        qv = [[decode(shards[w][t][j]) for j in range(qs)] for w in range(W)]
        kv = [[decode(shards[w][t][qs + j]) for j in range(ks)] for w in range(W)]
        ssq_q = sum((v * v for row in qv for v in row), Fraction(0))
        ssq_k = sum((v * v for row in kv for v in row), Fraction(0))
        dq = _dec(ssq_q / q_size + eps).sqrt()
        dk = _dec(ssq_k / kv_size + eps).sqrt()
        for w in range(W):
            q_out[w][t] = [_dec(qv[w][j]) / dq * _dec(decode(q_weight[w * qs + j]))
                           for j in range(qs)]
            k_out[w][t] = [_dec(kv[w][j]) / dk * _dec(decode(k_weight[w * ks + j]))
                           for j in range(ks)]
    return q_out, k_out
