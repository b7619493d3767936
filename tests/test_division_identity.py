"""The epilogues of both engines compute y32 = float(acc) / (s_x * s_w) as
RN_f32(double(a) * RN_f64(1 / double(d))) with a = float(acc) (or its bf16
rounding) and d the float32 product, instead of a float32 division per
element.  This is exactly the correctly rounded float32 quotient: a/d is a
quotient of two 24-bit floats, which is never a float32 rounding midpoint and
lies at least 2^-49 (relative) away from every one, while the double product
is within 2^-52 of a/d.  Checked here against numpy's IEEE float32 division
on random and adversarial pairs (host arithmetic, no GPU)."""

import numpy as np


def _double_rcp_quotient(a: np.ndarray, d: np.ndarray) -> np.ndarray:
    r = 1.0 / d.astype(np.float64)                # RN_f64(1/d)
    return (a.astype(np.float64) * r).astype(np.float32)


def _bf16(v: np.ndarray) -> np.ndarray:
    b = v.astype(np.float32).view(np.uint32).astype(np.uint64)
    return (((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32)


def test_random_accumulators_and_scales():
    rng = np.random.default_rng(4401)
    n = 2_000_000
    acc = np.where(rng.random(n) < 0.5, rng.integers(-3000, 3000, n), rng.integers(-(1 << 27), 1 << 27, n))
    a = acc.astype(np.float32)                    # float(acc): rounds beyond 2^24, as the kernels do
    d = ((rng.random(n) + 1.0) * np.exp2(rng.integers(-60, 80, n).astype(np.float64))).astype(np.float32)
    assert np.array_equal(_double_rcp_quotient(a, d).view(np.uint32), (a / d).view(np.uint32))
    ab = _bf16(a)                                 # the bf16-faithful numerator
    assert np.array_equal(_double_rcp_quotient(ab, d).view(np.uint32), (ab / d).view(np.uint32))


def test_adversarial_divisors():
    # all-ones significands, powers of two, and products of realistic scales
    rng = np.random.default_rng(4402)
    n = 500_000
    p2 = np.float32(2.0) ** rng.integers(-40, 40, n).astype(np.float32)
    ones = np.nextafter(p2, np.float32(0))
    s_x = (np.float32(127.0) / np.maximum(rng.random(n).astype(np.float32) * 20, np.float32(1e-5))).astype(np.float32)
    s_w = (np.float32(1.0) / np.maximum(rng.random(n).astype(np.float32) * 0.05, np.float32(1e-5))).astype(np.float32)
    acc = rng.integers(-(1 << 25), 1 << 25, n).astype(np.float32)
    for d in (p2, ones, (s_x * s_w).astype(np.float32)):
        assert np.array_equal(_double_rcp_quotient(acc, d).view(np.uint32), (acc / d).view(np.uint32))


def test_special_values():
    a = np.array([0.0, -0.0, 1.0, -1.0, 3.0, 16777217.0, -33554430.0], np.float32)
    d = np.array([1.0, 3.0, 0.0, 0.0, 1e-45, 7.0, 3.4e38], np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        want = a / d
        got = _double_rcp_quotient(a, d)
    same = (want.view(np.uint32) == got.view(np.uint32)) | (np.isnan(want) & np.isnan(got))
    assert same.all(), (want, got)
