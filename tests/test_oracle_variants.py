"""Pins of the oracle's variant rows: the single-level block constants ("QLoRA",
ozercemkelahmet.com, How it works, Step 2 without Step 3), the adapter-input
dropout and the gradient accumulation over micro-batches (the same page's code
example and training arguments)."""
import numpy as np
import pytest

from oracle import linear as olin
from oracle import nf4 as onf4
from synth import linear_problem


# ------------------------------------------------------------ single-level constants
def test_single_level_storage_is_half_a_bit_per_weight():
    # the page's figure: a 32-bit constant per 64 values is half a bit per weight
    for n in (64, 4096 * 4096, 11008 * 4096):
        codes, consts = onf4.storage_bytes_single_level(n)
        assert 8.0 * consts / n == 0.5
        assert 8.0 * (codes + consts) / n == 4.5
    assert onf4.storage_bytes_single_level(65) == (33, 8)


def _heavy_tail(n, seed):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    w[rng.random(n) < 1e-3] *= np.float32(8.0)
    return onf4.bf16_to_f32(onf4.f32_to_bf16_rn(w))


def test_single_level_codes_are_the_double_quant_codes():
    w = _heavy_tail(64 * 700 + 13, 1)
    a = onf4.quantize_single_level(w)
    b = onf4.quantize(w)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["absmax"], b["absmax"])


def test_single_level_round_trip_on_grid_values():
    # blocks made of bf16(L[c] * 2^k), each holding a +-1 level: absmax 2^k exactly,
    # so every value maps back to its level and dequantizes to itself
    L = onf4.nf4_levels()
    rng = np.random.default_rng(2)
    blocks = []
    for k in rng.integers(-12, 4, 40):
        c = rng.integers(0, 16, 64)
        c[rng.integers(0, 64)] = 15 if rng.random() < 0.5 else 0
        blocks.append((L[c] * np.float32(2.0 ** k)).astype(np.float32))
    w = onf4.bf16_to_f32(onf4.f32_to_bf16_rn(np.concatenate(blocks)))
    q = onf4.quantize_single_level(w)
    back = onf4.dequantize_single_level(q["codes"], q["absmax"], w.size)
    assert np.array_equal(back, onf4.f32_to_bf16_rn(w))


def test_single_level_equals_double_quant_where_the_constants_are_exact():
    # every block absmax = 255 * 2^k: step = 2^k and q8 = 255 reconstruct it exactly,
    # so both dequantizers must give the same bits
    rng = np.random.default_rng(3)
    k = -14
    a = np.float32(255.0 * 2.0 ** k)
    w = (rng.uniform(-1, 1, 64 * 256 * 2) * a).astype(np.float32)
    w = onf4.bf16_to_f32(onf4.f32_to_bf16_rn(w))
    w[::64] = a                                      # a representable bf16 value (255 has 8 bits)
    s = onf4.quantize_single_level(w)
    d = onf4.quantize(w)
    assert np.all(onf4.block_scales(d["q8"], d["step"]) == s["absmax"])
    assert np.array_equal(onf4.dequantize_single_level(s["codes"], s["absmax"], w.size),
                          onf4.dequantize(d["codes"], d["q8"], d["step"], w.size))


def test_single_level_error_bound():
    w = _heavy_tail(64 * 500, 4)
    q = onf4.quantize_single_level(w)
    deq = onf4.bf16_to_f32(onf4.dequantize_single_level(q["codes"], q["absmax"], w.size)).astype(np.float64)
    L = onf4.nf4_levels().astype(np.float64)
    half_gap = np.max(np.diff(L)) / 2
    a = np.repeat(q["absmax"].astype(np.float64), 64)
    v = np.abs(deq)
    _, e = np.frexp(v)
    half_ulp_bf16 = np.ldexp(1.0, np.maximum(e, -125) - 9)
    bound = a * half_gap + a * 2.0 ** -24 + half_ulp_bf16
    assert np.all(np.abs(deq - w) <= bound)


# ------------------------------------------------------------ adapter-input dropout
def _problem(M=6, N=16, K=32, r=4, seed=5):
    return linear_problem(M, N, K, r, 8.0, 0.02, seed=seed)


def test_dropout_with_everything_kept_is_the_plain_layer():
    p = _problem()
    keep = np.ones(p.X.shape)
    Y0, XA0 = olin.forward(p.X, p.W, p.A, p.B, 2.0)
    Y1, XA1 = olin.forward_dropout(p.X, p.W, p.A, p.B, 2.0, keep, 0.0)
    assert np.array_equal(Y0, Y1) and np.array_equal(XA0, XA1)
    g0 = olin.backward(p.dY, p.X, p.W, p.A, p.B, 2.0)
    g1 = olin.backward_dropout(p.dY, p.X, p.W, p.A, p.B, 2.0, keep, 0.0)
    for k in ("G", "dX", "dA", "dB"):
        assert np.array_equal(g0[k], g1[k])


def test_dropout_with_nothing_kept_leaves_the_frozen_path():
    p = _problem()
    keep = np.zeros(p.X.shape)
    Y, XA = olin.forward_dropout(p.X, p.W, p.A, p.B, 2.0, keep, 0.3)
    X = olin.as_f64(p.X)
    W = olin.as_f64(p.W)
    assert np.array_equal(Y, X @ W.T) and not XA.any()
    g = olin.backward_dropout(p.dY, p.X, p.W, p.A, p.B, 2.0, keep, 0.3)
    assert np.array_equal(g["dX"], olin.as_f64(p.dY) @ W)
    assert not g["dA"].any() and not g["dB"].any()


def test_dropout_backward_is_the_gradient_of_its_forward():
    p = _problem(M=4, N=8, K=16, r=2, seed=6)
    rng = np.random.default_rng(7)
    drop = 0.25
    keep = (rng.random(p.X.shape) >= drop).astype(np.float64)
    s = 2.0
    X, W, A, B, dY = (olin.as_f64(t) for t in (p.X, p.W, p.A, p.B, p.dY))

    def loss(X_, A_, B_):
        Y, _ = olin.forward_dropout(X_, W, A_, B_, s, keep, drop)
        return float(np.sum(Y * dY))

    g = olin.backward_dropout(dY, X, W, A, B, s, keep, drop)
    h = 1e-6
    for name, T, idx in (("dX", X, (1, 3)), ("dX", X, (2, 7)), ("dA", A, (5, 1)), ("dB", B, (1, 6))):
        Tp, Tm = T.copy(), T.copy()
        Tp[idx] += h
        Tm[idx] -= h
        args_p = [Tp if T is X else X, Tp if T is A else A, Tp if T is B else B]
        args_m = [Tm if T is X else X, Tm if T is A else A, Tm if T is B else B]
        fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert abs(fd - g[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_dropout_is_unbiased():
    p = _problem(M=3, N=5, K=24, r=4, seed=8)
    rng = np.random.default_rng(9)
    drop = 0.2
    Y_plain, _ = olin.forward(p.X, p.W, p.A, p.B, 2.0)
    ys = np.stack([olin.forward_dropout(p.X, p.W, p.A, p.B, 2.0,
                                        (rng.random(p.X.shape) >= drop).astype(np.float64), drop)[0]
                   for _ in range(4000)])
    se = ys.std(axis=0) / np.sqrt(len(ys))
    assert np.all(np.abs(ys.mean(axis=0) - Y_plain) <= 6 * se + 1e-12)


# ------------------------------------------------------------ gradient accumulation
@pytest.mark.parametrize("drop", [0.0, 0.1])
def test_accumulated_micro_batches_equal_the_full_batch(drop):
    p = linear_problem(12, 16, 32, 4, 8.0, 0.02, seed=10)
    rng = np.random.default_rng(11)
    keep = (rng.random(p.X.shape) >= drop).astype(np.float64)
    full = olin.backward_dropout(p.dY, p.X, p.W, p.A, p.B, 2.0, keep, drop)
    acc = None
    for lo, hi in ((0, 5), (5, 9), (9, 12)):
        g = olin.backward_dropout(p.dY[lo:hi], p.X[lo:hi], p.W, p.A, p.B, 2.0, keep[lo:hi], drop)
        acc = olin.accumulate_grads(acc, g)
    for k in ("dA", "dB"):
        assert np.allclose(acc[k], full[k], rtol=1e-12, atol=1e-14)
