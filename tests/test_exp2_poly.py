"""The FMA-pipe exponential of the forward kernel, checked on the CPU.

exp2_poly3 (exact_attention_117_b200/csrc/sm100.cuh) computes 2^x as
2^round(x) * p(x - round(x)) with a cubic p; the kernel uses it for one
exponential in four.  This test evaluates the same float32 steps in numpy and
bounds the relative error against 2^x; it also re-derives the coefficients
with the Remez script that produced them.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_117_b200", "csrc")


def _coeffs_from_source():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("float exp2_poly3"):]
    body = body[:body.index("}")]
    nums = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body)]
    # fmaxf bound, the 1.5*2^23 constant twice, then c3, c2, c1, c0
    c3, c2, c1, c0 = nums[3], nums[4], nums[5], nums[6]
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def exp2_poly3(x):
    c0, c1, c2, c3 = _coeffs_from_source()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = np.float32(c3) * f + c2
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_over_the_range_the_kernel_uses():
    x = np.linspace(-125.9, 8.0, 2_000_001, dtype=np.float32)
    y = exp2_poly3(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4      # bf16 rounding of P is 2^-9 = 2e-3
    assert np.all(y > 0)


def test_integer_arguments_are_nearly_exact_and_tiny_arguments_underflow():
    for n in range(-120, 9):
        assert abs(float(exp2_poly3(np.float32(n))) / 2.0 ** n - 1.0) < 1e-4
    assert float(exp2_poly3(np.float32(-1000.0))) <= 2.0 ** -125


def test_coefficients_match_the_remez_script():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.remez_exp2()
    assert err < 7.6e-5
    assert np.allclose(c, _coeffs_from_source(), rtol=0, atol=2e-6)
