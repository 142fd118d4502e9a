"""The polynomial exp2 that the FP8 softmax uses for a quarter of its scores
(exp2_poly3x2 in sm100_ptx.cuh), evaluated on the CPU with the kernel's own
constants read from the source: its error against the mathematical 2^y, its
exact values at integers, its range guard, and that the constants are the ones
the committed fit produces."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_ring_b200", "csrc")


def _constants():
    src = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = src[src.index("float2 exp2_poly3x2("):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    c3, c2, c1 = (np.float32(float.fromhex(h)) for h in dict.fromkeys(hexes))  # Horner order, deduplicated
    assert "make_float2(1.f, 1.f)" in body  # c0 = 1
    return np.float32(1.0), c1, c2, c3


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding to float32 after the add
    return (a.astype(np.float64) * b + c).astype(np.float32)


def _exp2_poly(y, c):
    """Step by step as the kernel does it, in float32."""
    c0, c1, c2, c3 = c
    shift = np.float32(12582912.0)
    y = np.maximum(y.astype(np.float32), np.float32(-126.0))
    t = (y + shift).astype(np.float32)
    jf = (t - shift).astype(np.float32)
    r = (y - jf).astype(np.float32)
    p = _fma32(r, c3, c2)
    p = _fma32(p, r, c1)
    p = _fma32(p, r, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    c = _constants()
    y = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = _exp2_poly(y, c).astype(np.float64)
    rel = np.abs(got / np.exp2(y.astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4, rel.max()
    # well inside a bf16 or E4M3 rounding step
    assert rel.max() < 2.0 ** -9 / 10


def test_exact_at_integers_and_guarded_below():
    c = _constants()
    j = np.arange(-126, 9).astype(np.float32)
    assert np.array_equal(_exp2_poly(j, c), np.exp2(j.astype(np.float64)).astype(np.float32))
    low = _exp2_poly(np.array([-126.5, -200.0, -1e30, -np.inf], dtype=np.float32), c)
    assert np.all(low >= 0) and np.all(low <= 2.0 ** -125)


def test_constants_come_from_the_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    coef, err = fit.fit(3)
    assert err < 1.02e-4
    assert np.allclose(coef, np.array(_constants(), dtype=np.float32), rtol=2e-6, atol=0)
