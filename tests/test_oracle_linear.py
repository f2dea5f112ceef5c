"""Pins for the fp64 linear-layer oracle: pure-Python loops on tiny shapes,
finite differences of the forward (which fixes the backward independently of
its formula), and the reductions the definition implies."""
import numpy as np

from oracle import linear, nf4
from synth import linear_problem, bf16_bits_to_f32


def _tiny(seed=0, M=3, N=5, K=7, r=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    A = rng.standard_normal((K, r))
    B = rng.standard_normal((r, N))
    dY = rng.standard_normal((M, N))
    return X, W, A, B, dY


def test_forward_matches_python_loops():
    X, W, A, B, _ = _tiny()
    s = 0.75
    M, K = X.shape
    N, r = W.shape[0], A.shape[1]
    Y, XA = linear.forward(X, W, A, B, s)
    for m in range(M):
        xa = [sum(X[m][k] * A[k][j] for k in range(K)) for j in range(r)]
        for j in range(r):
            assert abs(XA[m, j] - xa[j]) < 1e-12
        for n in range(N):
            y = sum(X[m][k] * W[n][k] for k in range(K)) + s * sum(xa[j] * B[j][n] for j in range(r))
            assert abs(Y[m, n] - y) < 1e-12


def test_backward_matches_python_loops():
    X, W, A, B, dY = _tiny(1)
    s = 1.5
    M, K = X.shape
    N, r = W.shape[0], A.shape[1]
    g = linear.backward(dY, X, W, A, B, s)
    G = [[sum(dY[m][n] * B[j][n] for n in range(N)) for j in range(r)] for m in range(M)]
    XA = [[sum(X[m][k] * A[k][j] for k in range(K)) for j in range(r)] for m in range(M)]
    for m in range(M):
        for k in range(K):
            v = sum(dY[m][n] * W[n][k] for n in range(N)) + s * sum(G[m][j] * A[k][j] for j in range(r))
            assert abs(g["dX"][m, k] - v) < 1e-12
    for k in range(K):
        for j in range(r):
            assert abs(g["dA"][k, j] - s * sum(X[m][k] * G[m][j] for m in range(M))) < 1e-12
    for j in range(r):
        for n in range(N):
            assert abs(g["dB"][j, n] - s * sum(XA[m][j] * dY[m][n] for m in range(M))) < 1e-12


def test_backward_is_gradient_of_forward():
    """Central differences of L = sum(dY * Y) w.r.t. X, A, B (Y is linear in each,
    so the differences are exact up to rounding).  No gradient reaches W."""
    X, W, A, B, dY = _tiny(2, M=2, N=4, K=5, r=3)
    s = 0.4
    g = linear.backward(dY, X, W, A, B, s)

    def loss(X_, A_, B_):
        return float(np.sum(dY * linear.forward(X_, W, A_, B_, s)[0]))

    h = 1e-3
    for name, T in (("dX", X), ("dA", A), ("dB", B)):
        num = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            args_p = {"dX": (Tp, A, B), "dA": (X, Tp, B), "dB": (X, A, Tp)}[name]
            args_m = {"dX": (Tm, A, B), "dA": (X, Tm, B), "dB": (X, A, Tm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-9, atol=1e-9)


def test_reductions():
    X, W, A, B, dY = _tiny(3)
    Y0, _ = linear.forward(X, W, A, B, 0.0)
    np.testing.assert_allclose(Y0, X @ W.T, rtol=1e-14, atol=1e-14)
    Yz, _ = linear.forward(X, W, np.zeros_like(A), B, 2.0)
    np.testing.assert_allclose(Yz, X @ W.T, rtol=1e-14, atol=1e-14)
    # linear in s
    Y1, _ = linear.forward(X, W, A, B, 1.0)
    Y3, _ = linear.forward(X, W, A, B, 3.0)
    np.testing.assert_allclose(Y3 - Y0, 3 * (Y1 - Y0), rtol=1e-12, atol=1e-12)
    g = linear.backward(dY, X, W, A, B, 0.0)
    assert np.all(g["dA"] == 0) and np.all(g["dB"] == 0)
    np.testing.assert_allclose(g["dX"], dY @ W, rtol=1e-14, atol=1e-14)


def test_bf16_inputs_and_sampled_rows():
    p = linear_problem(8, 128, 64, 8, 16.0, 0.02, seed=0)
    q = nf4.quantize_bf16(p.W)
    Wd = nf4.dequantize(q["codes"], q["q8"], q["step"], p.N * p.K).reshape(p.N, p.K)
    Y, XA = linear.forward(p.X, Wd, p.A, p.B, p.s)
    rows = np.array([1, 5])
    Yr, _ = linear.forward_rows(p.X, Wd, p.A, p.B, p.s, rows)
    np.testing.assert_allclose(Yr, Y[rows], rtol=1e-14, atol=1e-14)
    g = linear.backward(p.dY, p.X, Wd, p.A, p.B, p.s)
    dxr = linear.backward_rows_dx(p.dY, Wd, p.A, p.B, p.s, rows)
    np.testing.assert_allclose(dxr, g["dX"][rows], rtol=1e-14, atol=1e-14)
    # inputs really are the bf16 values
    assert np.array_equal(linear.as_f64(p.X), bf16_bits_to_f32(p.X).astype(np.float64))


def test_rel_fro():
    a = np.ones((3, 3))
    assert linear.rel_fro(a, a) == 0.0
    assert abs(linear.rel_fro(a * 1.001, a) - 1e-3) < 1e-12


def test_lora_products_match_full_backward():
    X, W, A, B, dY = _tiny(4)
    s = 1.25
    lp = linear.lora_products(dY, X, A, B, s)
    g = linear.backward(dY, X, W, A, B, s)
    _, XA = linear.forward(X, W, A, B, s)
    np.testing.assert_allclose(lp["XA"], XA, rtol=1e-14, atol=1e-14)
    for k in ("G", "dA", "dB"):
        np.testing.assert_allclose(lp[k], g[k], rtol=1e-13, atol=1e-13)
