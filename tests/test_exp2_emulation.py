"""The FMA-pipe 2^x of the tensor-core attention kernels (ex2_poly2 in
h2o_kv_cache_b200/csrc/attn_common.cuh), checked on the CPU.

The kernels take a quarter of their exponentials from a Cody-Waite range
reduction and a cubic instead of the MUFU unit.  This test reads the cubic's
coefficients from the CUDA source, replays the kernel's fp32 operation sequence
bit for bit (fmaxf clamp, an add rounded towards -inf, exact subtractions, fused
multiply-adds, an integer add on the exponent bits), and checks it against the
exact 2^x: the relative error bound the design relies on, and that masked (-inf),
NaN and very negative inputs give a tiny non-negative value, never NaN or inf.
"""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "h2o_kv_cache_b200", "csrc", "attn_common.cuh")


def _coefficients():
    src = open(SRC).read()
    body = src[src.index("void ex2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = [float(x) for x in re.findall(r"f2_pack\(([0-9.eE+-]+)f, \1f\)", body)]
    # the magic constant first, then c3, c2, c1, c0 in Horner order
    assert lits[0] == 12582912.0, lits
    c3, c2, c1, c0 = lits[1:5]
    return c0, c1, c2, c3


def _add_rm(a, b):
    exact = a.astype(np.float64) + np.float64(b)
    r = exact.astype(np.float32)
    over = r.astype(np.float64) > exact
    r[over] = np.nextafter(r[over], np.float32(-np.inf))
    return r


def _fma(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding of the sum
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _ex2_poly(x, coef):
    c0, c1, c2, c3 = (np.float32(c) for c in coef)
    x = np.fmax(x.astype(np.float32), np.float32(-126.0))          # fmaxf: NaN -> -126
    t = _add_rm(x, 12582912.0)                                        # 1.5 * 2^23 + floor(x)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)         # exact, in [0, 1)
    ones = np.ones_like(f)
    q = _fma(_fma(_fma(ones * c3, f, ones * c2), f, ones * c1), f, ones * c0)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_bound():
    coef = _coefficients()
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-125.0, 0.5, 2_000_000), np.linspace(-2.0, 0.0, 200_001),
                        -np.arange(0, 126, dtype=np.float64)]).astype(np.float32)
    y = _ex2_poly(x, coef).astype(np.float64)
    rel = y / np.exp2(x.astype(np.float64)) - 1.0
    assert np.abs(rel).max() < 8e-5
    assert abs(rel.mean()) < 2e-5          # no bias that would shift summed weights


def test_masked_and_out_of_range_inputs_are_tiny_and_finite():
    coef = _coefficients()
    x = np.array([-np.inf, np.nan, -126.0, -126.5, -127.0, -1e30, -3e38], dtype=np.float32)
    y = _ex2_poly(x, coef)
    assert np.all(np.isfinite(y)) and np.all(y >= 0.0)
    assert np.all(y <= np.float32(2.0 ** -125))


@pytest.mark.parametrize("x", [0.0, -1.0, -0.5, -10.25, -100.75])
def test_exact_points(x):
    coef = _coefficients()
    y = float(_ex2_poly(np.array([x], dtype=np.float32), coef)[0])
    assert abs(y / 2.0 ** x - 1.0) < 8e-5
