"""GPU parity of the single-level block constants ("QLoRA", ozercemkelahmet.com,
How it works, Step 2 without Step 3: one fp32 constant per 64 values, half a bit
per weight) against the oracle (oracle.nf4.quantize_single_level /
dequantize_single_level): codes and constants bit-exact, dequant bit-exact (the
standalone kernel, inside both fused GEMMs, inside the few-token kernel and in
the merge), and the linear layer within the bars of the double-quant weight."""
import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from oracle import nf4 as onf4
from synth import linear_problem, normal_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 100), (128, 4096), (257, 1000), (1024, 16384 + 64)])
def test_single_level_quantize_and_dequant_bit_exact(q, rows, cols):
    bits = normal_bf16(7, f"sl{rows}x{cols}", (rows, cols), 0.02)
    Wq = q.nf4_quantize(H.bits_to_dev(bits, (rows, cols)), single_level=True)
    assert Wq.q8 is None and q.device_status() == (0, 0)
    ref = onf4.quantize_single_level(onf4.bf16_to_f32(bits.ravel()))
    assert np.array_equal(Wq.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(Wq.step.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    got = H.dev_to_bits(q.nf4_dequant(Wq)).ravel()
    assert np.array_equal(got, onf4.dequantize_single_level(ref["codes"], ref["absmax"], bits.size))


def _single_deq_bits(W_bits):
    ref = onf4.quantize_single_level(onf4.bf16_to_f32(W_bits.ravel()))
    return onf4.dequantize_single_level(ref["codes"], ref["absmax"], W_bits.size).reshape(W_bits.shape)


@pytest.mark.parametrize("M,N,K,r", [(300, 384, 256, 16), (16, 1024, 1024, 8), (1, 256, 512, 16),
                                     (513, 256, 384, 64), (300, 12800, 256, 16)])
def test_single_level_linear(q, M, N, K, r):
    import torch
    p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=3)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W), single_level=True)
    Y, XA = q.linear_fwd(X, Wq, A, B, p.s)
    dX, dA, dB = q.linear_bwd(dY, X, XA, Wq, A, B, p.s)
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    Wd = _single_deq_bits(p.W)
    Yr, XAr = olin.forward(p.X, Wd, p.A, p.B, p.s)
    g = olin.backward(p.dY, p.X, Wd, p.A, p.B, p.s)
    Yb, dXb = H.dev_to_bits(Y), H.dev_to_bits(dX)
    assert olin.rel_fro(onf4.bf16_to_f32(Yb), Yr) <= 2e-3
    assert olin.rel_fro(onf4.bf16_to_f32(dXb), g["dX"]) <= 2e-3
    assert H.bf16_ulp_check(Yb, Yr, K + 2 * r) <= 1.0
    assert H.bf16_ulp_check(dXb, g["dX"], N + 2 * r) <= 1.0
    mag = H.lora_magnitudes(p.X, p.A, p.B, p.dY, p.s, XA=XAr)
    for name, got, ref in (("XA", XA, XAr), ("dA", dA, g["dA"]), ("dB", dB, g["dB"])):
        got = got.cpu().numpy().astype(np.float64)
        assert olin.rel_fro(got, ref) <= 1e-4, name
        assert H.mag_check(got, ref, mag[name]) <= 1.0, name


@pytest.mark.parametrize("N,K", [(256, 384), (384, 256)])
def test_single_level_gemm_dequant_bit_exact_one_hot(q, N, K):
    """One-hot tokens pick single weights in both fused GEMMs (A = 0): Y = deq(W)^T
    and dX = deq(W) bit for bit with single-level constants."""
    import torch
    Wb = normal_bf16(2, f"slonehot{N}x{K}", (N, K), 0.02)
    ref = _single_deq_bits(Wb)
    Wq = q.nf4_quantize(H.bits_to_dev(Wb), single_level=True)
    r = 16
    A = torch.zeros(K, r, dtype=torch.bfloat16, device="cuda")
    B = torch.randn(r, N, device="cuda").to(torch.bfloat16)
    Y, _ = q.linear_fwd(torch.eye(K, dtype=torch.bfloat16, device="cuda"), Wq, A, B, 2.0)
    dX, _, _ = q.linear_bwd(torch.eye(N, dtype=torch.bfloat16, device="cuda"),
                            torch.zeros(N, K, dtype=torch.bfloat16, device="cuda"), None, Wq, A, B, 2.0)
    torch.cuda.synchronize()
    assert np.array_equal(H.dev_to_bits(Y), ref.T)
    assert np.array_equal(H.dev_to_bits(dX), ref)


def test_single_level_few_token_dequant_bit_exact(q):
    import torch
    N, K = 256, 512
    Wb = normal_bf16(4, "slsk", (N, K), 0.02)
    ref = _single_deq_bits(Wb)
    Wq = q.nf4_quantize(H.bits_to_dev(Wb), single_level=True)
    A = torch.zeros(K, 16, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(16, N, dtype=torch.bfloat16, device="cuda")
    for start in range(0, K, 16):
        X = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
        X[torch.arange(16), torch.arange(start, start + 16)] = 1.0
        Y, _ = q.linear_fwd(X, Wq, A, B, 1.0)
        torch.cuda.synchronize()
        assert np.array_equal(H.dev_to_bits(Y), ref[:, start:start + 16].T), start


def test_single_level_merge_base_is_the_dequant(q):
    import torch
    p = linear_problem(1, 256, 512, 16, 32.0, 0.02, seed=5, with_dy=False)
    Wq = q.nf4_quantize(H.bits_to_dev(p.W), single_level=True)
    out = q.nf4_merge(H.bits_to_dev(p.A), torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda"), 2.0, Wq=Wq)
    torch.cuda.synchronize()
    assert np.array_equal(H.dev_to_bits(out), _single_deq_bits(p.W))
