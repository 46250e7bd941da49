"""The FMA-pipe exp2 of the kernels (ex2_fma in csrc/common.cuh), emulated
step by step in IEEE float32 on the host and held to the exact 2^x: Cody and
Waite's range reduction with the 1.5 * 2^23 rounding constant, the degree-5
polynomial fitted by Lawson's method, and the exponent-field add.  The device
routine itself is exercised by the GPU selection tests, whose scores sum its
results."""
import re
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coefficients():
    # read the constants the device routine uses, highest degree first
    src = open(os.path.join(ROOT, "token_level_top_hs2_b200", "csrc", "common.cuh")).read()
    body = src[src.index("HS2_DEV float ex2_fma"):]
    body = body[:body.index("\n}\n")]
    first = re.search(r"float p = ([-+0-9.e]+)f;", body).group(1)
    rest = re.findall(r"p = fmaf\(p, f, ([-+0-9.e]+)f\);", body)
    return [np.float32(first)] + [np.float32(c) for c in rest]


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding of the sum to
    # float64, then to float32 (a double rounding only on exact ties of the
    # float64 result, far rarer than the tolerance below cares about)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma_emulated(x):
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    big = np.float32(12582912.0)
    t = (xc + big).astype(np.float32)
    n = (t - big).astype(np.float32)
    f = (xc - n).astype(np.float32)
    cs = _coefficients()
    p = np.full_like(f, cs[0])
    for c in cs[1:]:
        p = _fma32(p, f, np.full_like(f, c))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_six_coefficients_near_the_taylor_series():
    cs = _coefficients()[::-1]  # constant term first
    assert len(cs) == 6
    ln2 = np.log(2.0)
    taylor = [ln2 ** i / np.prod(np.arange(1, i + 1)) for i in range(6)]
    for c, tc in zip(cs, taylor):
        assert abs(c - tc) <= 0.02 * tc


def test_relative_error_against_exact_exp2():
    x = np.concatenate([np.linspace(-125.0, 4.0, 400001, dtype=np.float32),
                        np.float32(-np.arange(0, 126)), np.float32(np.arange(0, 5)),
                        np.float32(-np.arange(0, 126)) + np.float32(0.5)])
    got = ex2_fma_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= 2.5e-7, float(rel.max())


def test_below_the_clamp_stays_tiny_and_positive():
    x = np.array([-126.0, -150.0, -1e6, -np.inf], dtype=np.float32)
    got = ex2_fma_emulated(x)
    assert np.all(got > 0) and np.all(got <= np.float32(2.0 ** -124))


def test_integer_inputs_are_exact_powers_of_two():
    # f = 0 there: the polynomial gives 1.0000001, so 2^n within one ulp
    x = np.float32(-np.arange(0, 126))
    got = ex2_fma_emulated(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) <= 2 ** -23)
