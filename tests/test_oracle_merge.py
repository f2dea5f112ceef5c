"""Pins of the merge-path oracle (the adapter folded into a 16-bit weight,
"QLoRA", ozercemkelahmet.com, How it works, Step 8 and section "Merging after
QLoRA") and of the one-step fp64 -> bf16 rounding it ends with.

The rounding is pinned by an exact-rational nearest search over the bf16
neighbours; the merge by exact rational arithmetic on tiny shapes, by its
reduction to the base weight, and by the equivalence it exists for: the merged
weight's forward equals the adapted forward up to the one rounding."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import linear as olin
from oracle import nf4 as onf4
from synth import linear_problem


def _bf16_value(bits: int) -> Fraction:
    return Fraction(float(onf4.bf16_to_f32(np.array([bits], np.uint16))[0]))


def _nearest_bf16(exact: Fraction, guess: int) -> int:
    """Nearest bf16 (ties to even bits) to an exact rational, searching the finite
    bf16 values of the guess's sign around the guess (and the zero of that sign,
    which is what IEEE rounding gives a tiny value)."""
    sign = guess & 0x8000
    mag = guess & 0x7FFF
    cands = {sign | max(0, min(0x7F7F, mag + d)) for d in (-2, -1, 0, 1, 2)} | {sign}
    best = None
    for c in sorted(cands):
        d = abs(exact - _bf16_value(c))
        key = (d, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_one_rounding_matches_exact_nearest_search():
    rng = np.random.default_rng(5)
    mant = rng.uniform(-1, 1, 6000)
    expo = rng.integers(-140, 60, 6000)
    x = np.ldexp(mant, expo)                        # normal and bf16-subnormal magnitudes
    got = onf4.f64_to_bf16_rn(x)
    guess = onf4.f32_to_bf16_rn(x.astype(np.float32))
    for xi, g, q in zip(x, got, guess):
        assert int(g) == _nearest_bf16(Fraction(float(xi)), int(q)), float(xi)


def test_one_rounding_on_exact_ties_and_their_neighbours():
    rng = np.random.default_rng(6)
    bits = rng.integers(0x0001, 0x7F7F, 3000).astype(np.uint16)
    bits |= (rng.integers(0, 2, 3000).astype(np.uint16) << np.uint16(15))
    lo = onf4.bf16_to_f32(bits).astype(np.float64)
    hi = onf4.bf16_to_f32((bits & 0x8000) | ((bits & 0x7FFF) + 1)).astype(np.float64)
    mid = (lo + hi) / 2                              # exact in fp64
    even_is_lo = (bits & 1) == 0
    want_tie = np.where(even_is_lo, bits, (bits & 0x8000) | ((bits & 0x7FFF) + 1))
    assert np.array_equal(onf4.f64_to_bf16_rn(mid), want_tie.astype(np.uint16))
    away = np.nextafter(mid, np.copysign(np.inf, mid))
    toward = np.nextafter(mid, 0.0)
    assert np.array_equal(onf4.f64_to_bf16_rn(away), ((bits & 0x8000) | ((bits & 0x7FFF) + 1)).astype(np.uint16))
    assert np.array_equal(onf4.f64_to_bf16_rn(toward), bits)


def test_one_rounding_differs_from_two_where_it_must():
    # 1 + 2^-8 + 2^-30 lies above the bf16 tie 1 + 2^-8; via fp32 it lands on the tie
    # and then rounds to even (1.0).  One rounding gives 1 + 2^-7.
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -30, -(1 + 2.0 ** -8 + 2.0 ** -30)])
    assert list(onf4.f64_to_bf16_rn(x)) == [0x3F81, 0xBF81]
    assert list(onf4.f32_to_bf16_rn(x.astype(np.float32))) == [0x3F80, 0xBF80]


def test_one_rounding_special_values():
    x = np.array([0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 3.3e38, 3.4e38, -3.4e38])
    assert list(onf4.f64_to_bf16_rn(x)) == [0x0000, 0x8000, 0x0001, 0x0000, 0x0001, 0x7F78, 0x7F80, 0xFF80]


def test_one_rounding_agrees_with_the_fp32_helper_on_fp32_values():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(0.05)
    assert np.array_equal(onf4.f64_to_bf16_rn(x.astype(np.float64)), onf4.f32_to_bf16_rn(x))


def _exact_merge_bits(Wb, A, B, s):
    N, K = Wb.shape
    r = A.shape[1]
    out = np.zeros((N, K), np.uint16)
    fs = Fraction(float(s))
    for n in range(N):
        for k in range(K):
            v = _bf16_value(int(Wb[n, k]))
            for j in range(r):
                v += fs * _bf16_value(int(A[k, j])) * _bf16_value(int(B[j, n]))
            guess = int(onf4.f32_to_bf16_rn(np.array([float(v)], np.float32))[0])
            out[n, k] = _nearest_bf16(v, guess)
    return out


@pytest.mark.parametrize("seed", [0, 1])
def test_merge_exact_rational_on_tiny_shapes(seed):
    p = linear_problem(2, 6, 5, 3, 6.0, 0.02, seed=seed)
    got = olin.merge_weight(p.W, p.A, p.B, 2.0)
    assert np.array_equal(got, _exact_merge_bits(p.W, p.A, p.B, 2.0))


def test_merge_without_adapter_is_the_base_weight():
    p = linear_problem(4, 64, 128, 8, 16.0, 0.02, seed=3)
    wb = onf4.bf16_to_f32(p.W)
    zeroB = np.zeros_like(p.B)
    for got in (olin.merge_weight(p.W, p.A, zeroB, 2.0), olin.merge_weight(p.W, p.A, p.B, 0.0)):
        assert np.array_equal(onf4.bf16_to_f32(got), wb)     # values (a -0 base gives +0)


def _half_quantum(bits):
    v = np.abs(onf4.bf16_to_f32(bits).astype(np.float64))
    _, e = np.frexp(v)
    e = np.maximum(np.where(v > 0, e, -125), -125)
    return np.ldexp(1.0, e - 9)


def _merged_forward_gap(p, Wb_bits, merged_bits, s):
    X = onf4.bf16_to_f32(p.X).astype(np.float64)
    Y_merged = X @ onf4.bf16_to_f32(merged_bits).astype(np.float64).T
    Y_adapter, _ = olin.forward(p.X, Wb_bits, p.A, p.B, s)
    bound = np.abs(X) @ _half_quantum(merged_bits).T
    return np.abs(Y_merged - Y_adapter), bound


@pytest.mark.parametrize("base", ["bf16 original", "dequantized NF4"])
def test_merged_forward_equals_the_adapted_forward(base):
    p = linear_problem(7, 48, 256, 8, 16.0, 0.02, seed=4)
    s = 16.0 / 8
    if base == "bf16 original":
        Wb = p.W
    else:
        q = onf4.quantize_bf16(p.W.ravel())
        Wb = onf4.dequantize(q["codes"], q["q8"], q["step"], p.W.size).reshape(p.W.shape)
    merged = olin.merge_weight(Wb, p.A, p.B, s)
    gap, bound = _merged_forward_gap(p, Wb, merged, s)
    assert np.all(gap <= bound * (1 + 1e-9) + 1e-12)
    # the bound is tight enough to catch a wrong sign or scale of the adapter term
    wrong = olin.merge_weight(Wb, p.A, p.B, -s)
    gap, bound = _merged_forward_gap(p, Wb, wrong, s)
    assert np.any(gap > 10 * bound)
