"""The causal prefill's FMA-pipe exp2 (one key pair in four skips ex2.approx): its
constants, read from the kernel source, and its fp32 steps emulated here, against 2^d.

The softmax of "Tensor Product Attention Is All You Need" (arXiv:2501.06425, §3.1) takes
exp of the scaled scores; the kernel works in base 2 (the log2(e) factor is folded into
the score scale), so every p is 2^d with d <= 8 after the running max is subtracted.  P is
rounded to bf16 for the value product, whose half-ulp is 2^-9 relative: the
approximation must stay well inside that."""
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "tensor_product_attention_b200" / "csrc" / "prefill_qm.cu"


def _constants():
    text = SRC.read_text()
    m = re.search(r"kE2C0 = ([0-9.e+-]+)f, kE2C1 = ([0-9.e+-]+)f, kE2C2 = ([0-9.e+-]+)f, kE2C3 = ([0-9.e+-]+)f",
                  text)
    assert m, "exp2 polynomial constants not found in the prefill kernel"
    return [np.float32(float(v)) for v in m.groups()]


def _fma32(a, b, c):
    # fp32 fused multiply-add: exact product and sum in fp64, one rounding to fp32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma(d):
    """The kernel's steps, in fp32 with its integer exponent update."""
    c0, c1, c2, c3 = _constants()
    shift = np.float32(12582912.0)
    d = np.maximum(d.astype(np.float32), np.float32(-126.0))
    t = (d + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), d)
    q = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    # every d the softmax meets after the max subtraction (<= 8 with the lazy rescale),
    # densely, including the half-integers where the rounding of n changes
    d = np.concatenate([np.linspace(-125.0, 9.0, 400001), np.arange(-125, 10) + 0.5,
                        np.arange(-125, 10).astype(np.float64)]).astype(np.float32)
    got = ex2_fma(d).astype(np.float64)
    ref = np.exp2(d.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 20


def test_exact_at_zero_and_monotone_near_the_max():
    # the row's max element has d = 0: p must be ~1 (it anchors the row sum)
    assert abs(float(ex2_fma(np.array([0.0], np.float32))[0]) - 1.0) < 1e-4
    d = np.linspace(-4.0, 0.0, 20001).astype(np.float32)
    p = ex2_fma(d)
    assert np.all(np.diff(p.astype(np.float64)) >= -1e-7)


def test_underflow_clamp_stays_tiny_and_positive():
    # masked keys are zeroed explicitly in the kernel; other far-below-max terms are
    # clamped at 2^-126 and must neither wrap the exponent field nor turn negative
    d = np.array([-126.0, -200.0, -1e30, -np.inf], np.float32)
    p = ex2_fma(d).astype(np.float64)
    assert np.all(p >= 0.0) and np.all(p <= 2.0 ** -125)


def test_a_planted_coefficient_error_is_caught():
    # the 1e-4 bound above fails if a coefficient is off by 1% (planted here)
    c0, c1, c2, c3 = _constants()
    f = np.linspace(-0.5, 0.5, 10001)
    good = ((c3 * f + c2) * f + c1) * f + c0
    bad = ((c3 * f + c2 * 1.01) * f + c1) * f + c0
    ref = np.exp2(f)
    assert np.abs(good / ref - 1).max() < 1e-4
    assert np.abs(bad / ref - 1).max() > 1e-4
