"""Error bound of the FMA-pipe exp2 used for part of the softmax
exponentials (exp2_poly2 in csrc/sm100_ptx.cuh).

The device arithmetic is replayed step by step in IEEE fp32 with numpy (same
clamp, same 1.5 * 2^23 rounding shift, same Horner order with fused
multiply-adds emulated in float64 and rounded once to fp32, same integer
exponent insertion), with the coefficients read from the header itself, and
compared with the exact 2^x.  The bound: relative error <= 2e-4 (bf16 P
needs 2^-9 = 2e-3), exact +0 for x <= -127 and for -inf.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "attention_flash_attn_02_b200", "csrc", "sm100_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("exp2_poly2(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    lits = [float(x) for x in re.findall(r"f2\(([0-9.eE+-]+)f, \1f\)", body)]
    # order of appearance: c3, c2 (first fma), c1, then 1.0
    c3, c2, c1, one = lits[-4:]
    assert one == 1.0
    return np.float32(c1), np.float32(c2), np.float32(c3)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_emulated(x):
    c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    r = (t + (-shift)).astype(np.float32)
    f = _fma32(r, np.full_like(r, -1.0), x)
    p = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, 1.0))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound_over_softmax_range():
    # scores after subtracting the running max lie in [-inf, 8] (lazy rescale)
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 1_000_000))])
    y = exp2_poly_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 2e-4, rel.max()


def test_masked_and_underflow_give_exact_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.0], dtype=np.float32)
    y = exp2_poly_emulated(x)
    assert np.all(y == 0.0) and not np.any(np.signbit(y))


def test_integers_are_exact():
    k = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_array_equal(exp2_poly_emulated(k), np.exp2(k.astype(np.float64)).astype(np.float32))


def test_monotone_non_negative_near_underflow():
    x = np.linspace(-127.0, -120.0, 10001, dtype=np.float32)
    y = exp2_poly_emulated(x)
    assert np.all(y >= 0) and np.all(np.isfinite(y))
