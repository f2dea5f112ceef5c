"""GPU parity of the few-token forward (M <= 16 tokens; one cluster launch with
the NF4 weight decoded in registers) against the fp64 oracle.

Bars as in test_gpu_linear: relative Frobenius <= 2e-3 for Y (bf16 output) and
<= 1e-4 for the fp32 XA; Y also element-wise within one bf16 ulp (plus the
accumulation floor for near-zero results), XA element-wise within 2^-15 of
|X| |A|.  The dequantization inside the
kernel is checked bit for bit with one-hot tokens."""
import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from synth import linear_problem, normal_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _fwd(q, p):
    import torch
    X = H.bits_to_dev(p.X)
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    Y, XA = q.linear_fwd(X, Wq, H.bits_to_dev(p.A), H.bits_to_dev(p.B), p.s)
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    return H.dev_to_bits(Y), XA.cpu().numpy().astype(np.float64)


def _check(p, Yb, XA):
    Wd = H.oracle_deq_bits(p.W)
    Y, XAr = olin.forward(p.X, Wd, p.A, p.B, p.s)
    ey = olin.rel_fro(H.onf4.bf16_to_f32(Yb), Y)
    ex = olin.rel_fro(XA, XAr)
    assert ey <= 2e-3 and ex <= 1e-4, (ey, ex)
    assert H.bf16_ulp_check(Yb, Y, p.K + p.r) <= 1.0
    mag = np.abs(olin.as_f64(p.X)) @ np.abs(olin.as_f64(p.A))
    assert H.mag_check(XA, XAr, mag) <= 1.0
    return ey, ex


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K,r", [(256, 512, 16), (384, 640, 8), (256, 1024, 128), (128, 128, 24)])
def test_skinny_forward(q, M, N, K, r):
    p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=M)
    Yb, XA = _fwd(q, p)
    _check(p, Yb, XA)


@pytest.mark.parametrize("N", [4096, 11008])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_skinny_forward_decode_shapes(q, M, N):
    """The few-token workload at full size: W N x 4096, r = 16, full Y checked."""
    p = linear_problem(M, N, 4096, 16, 32.0, 0.02, seed=0, with_dy=False)
    Yb, XA = _fwd(q, p)
    _check(p, Yb, XA)


@pytest.mark.parametrize("N,K", [(256, 512), (128, 1024), (384, 640)])
def test_skinny_dequant_bit_exact_one_hot(q, N, K):
    """Tokens that are one-hot in K pick single weight columns: Y[m, n] =
    deq(W)[n, k_m] exactly, so the in-register decode must equal the oracle's
    dequantized bf16 bit for bit."""
    import torch
    Wb = normal_bf16(1, f"skonehot{N}x{K}", (N, K), 0.02)
    ref = H.oracle_deq_bits(Wb)
    Wq = q.nf4_quantize(H.bits_to_dev(Wb))
    r = 16
    A = torch.zeros(K, r, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(r, N, dtype=torch.bfloat16, device="cuda")
    for start in range(0, K, 16):
        ks = np.arange(start, min(K, start + 16))
        X = torch.zeros(len(ks), K, dtype=torch.bfloat16, device="cuda")
        X[torch.arange(len(ks)), torch.from_numpy(ks)] = 1.0
        Y, _ = q.linear_fwd(X, Wq, A, B, 1.0)
        torch.cuda.synchronize()
        assert np.array_equal(H.dev_to_bits(Y), ref[:, ks].T), start


@pytest.mark.parametrize("M", [1, 7, 16])
@pytest.mark.parametrize("N,K,r", [(256, 11008, 16), (128, 16384, 128), (128, 22016, 64)])
def test_skinny_forward_long_k(q, M, N, K, r):
    """Long contractions: cluster slices that stage A in several passes, and
    16-CTA clusters when an 8-way split does not fit in shared memory."""
    p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=M + 100, with_dy=False)
    Yb, XA = _fwd(q, p)
    _check(p, Yb, XA)


def test_few_tokens_beyond_skinny_plan(q):
    """A contraction too long for the one-launch plan still gives the right
    answer (the general fused path takes it)."""
    p = linear_problem(3, 128, 65536, 8, 16.0, 0.02, seed=5, with_dy=False)
    Yb, XA = _fwd(q, p)
    _check(p, Yb, XA)


@pytest.mark.parametrize("M,D,r", [(1, 4096, 16), (4, 2048, 64), (16, 1024, 8)])
def test_skinny_dependent_chain(q, M, D, r):
    """Consecutive few-token calls where each call's X is the previous call's Y (square
    weights, so the shapes chain).  Back-to-back on one stream, and replayed from a CUDA
    graph, the outputs equal those of calls separated by a device synchronize, bit for
    bit: a call reads its X only after the previous call's weight pass has finished,
    although its own weight pass may launch before that."""
    import torch
    layers = []
    for i in range(6):
        p = linear_problem(M, D, D, r, 2.0 * r, 0.02, seed=100 + i, with_dy=False)
        layers.append((q.nf4_quantize(H.bits_to_dev(p.W)), H.bits_to_dev(p.A), H.bits_to_dev(p.B), p.s))
    X0 = H.bits_to_dev(linear_problem(M, D, D, r, 2.0 * r, 0.02, seed=99, with_dy=False).X)
    ws = q.make_workspace(M, D, D, r, X0.device)
    outs = [torch.empty(M, D, dtype=torch.bfloat16, device="cuda") for _ in layers]

    def chain(sync):
        x = X0
        for (Wq, A, B, s), Y in zip(layers, outs):
            q.linear_fwd(x, Wq, A, B, s, workspace=ws, Y=Y, want_xa=False)
            if sync:
                torch.cuda.synchronize()
            x = Y

    chain(True)
    ref = [o.clone() for o in outs]
    for o in outs:
        o.zero_()
    chain(False)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(outs, ref))
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain(False)
    g.replay()
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    assert all(torch.equal(a, b) for a, b in zip(outs, ref))
