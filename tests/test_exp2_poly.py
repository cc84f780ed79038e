"""The polynomial 2^x the attention kernel uses for a quarter of its
exponentials: its coefficients are the ones the fit script produces, and the
algorithm (round-to-nearest split, degree-4 polynomial, exponent add),
emulated step by step in float32, stays within 4e-6 relative error of 2^x."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CU = os.path.join(ROOT, "full_gqa_learned_b200", "csrc", "flint_attn.cu")
FIT = os.path.join(ROOT, "full_gqa_learned_b200", "csrc", "exp2_poly_fit.py")


def coeffs_in_kernel():
    src = open(CU).read()
    return [np.float32(float(v)) for v in
            re.findall(r"constexpr float kExp2C\d = ([-0-9.e+]+)f;", src)]


def test_kernel_coefficients_match_fit_script():
    out = subprocess.run([sys.executable, FIT], capture_output=True, text=True, check=True).stdout
    fit = [np.float32(float(v)) for v in re.findall(r"= ([-0-9.e+]+)f;", out)]
    assert len(fit) == 5 and fit == coeffs_in_kernel()


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_poly(x, c):
    x = np.maximum(np.float32(x), np.float32(-126.0))
    sh = np.float32(12582912.0)
    t = np.float32(x + sh)
    n = np.float32(t - sh)
    f = np.float32(x - n)
    q = fma32(c[4], f, c[3])
    q = fma32(q, f, c[2])
    q = fma32(q, f, c[1])
    q = fma32(q, f, c[0])
    # the kernel adds bits(t) << 23 modulo 2^32, which equals n << 23 because
    # 0x4B400000 << 23 vanishes modulo 2^32
    tb = t.view(np.uint32).astype(np.uint64)
    bits = (q.view(np.uint32).astype(np.uint64) + (tb << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    ni = t.view(np.int32).astype(np.int64) - 0x4B400000
    ref_bits = (q.view(np.int32).astype(np.int64) + (ni << 23)) & 0xFFFFFFFF
    assert np.array_equal(bits.astype(np.int64), ref_bits)
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    c = coeffs_in_kernel()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125.0, 8.0, 200000), np.linspace(-2, 2, 40001),
                        np.arange(-125, 9)]).astype(np.float32)
    got = exp2_poly(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 4e-6
    assert exp2_poly(np.float32(0.0), c) == np.float32(1.0) or abs(exp2_poly(np.float32(0.0), c) - 1) < 1e-6
