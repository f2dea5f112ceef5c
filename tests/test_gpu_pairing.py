"""The two shapes of the fused GEMM launch, CTA pairs (256-row weight tiles over two
CTAs, for output widths that are multiples of 256) and single CTAs (128-row tiles),
each against the fp64 oracle, and against each other.

The bar per shape is that of the linear tests (bf16 outputs within one bf16 ulp
of the exact value, fp32 outputs within 2^-15 of their magnitude products).  The
two shapes accumulate each output over the same K steps in the same order, except
where the last-wave split (which depends on the number of units) divides a tile's
contraction into two halves summed in fp32; there their Y and dX may differ by the
rounding of two correct results (two units of the oracle bound), and on shapes with
no split they do not differ at all."""
import numpy as np
import pytest

import helpers as H
import test_gpu_linear as TL
from synth import linear_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _both(q, p):
    prev = q.set_gemm_pairing(True)
    try:
        on = TL._run(q, p)
        q.set_gemm_pairing(False)
        off = TL._run(q, p)
    finally:
        q.set_gemm_pairing(prev)
    return on, off


def _apart(a, b, contraction):
    """0 when the two bf16 arrays are identical; otherwise their largest distance in
    units of (one bf16 ulp + the fp32 accumulation floor of a `contraction`-term sum),
    as the oracle bound measures it.  Each side is within one such unit of the exact
    value, so two correct results are within two of each other."""
    if np.array_equal(a, b):
        return 0.0
    return H.bf16_ulp_check(a, H.onf4.bf16_to_f32(b).astype(np.float64), contraction)


# (M, N, K, r, alpha, split in either shape)
@pytest.mark.parametrize("M,N,K,r,alpha,split", [
    (300, 512, 768, 16, 32.0, False),     # fwd pairs (N = 512), dX pairs (K = 768), ragged tokens
    (513, 768, 512, 64, 16.0, False),     # r = 64: two LoRA stages on both CTAs of a pair
    (257, 256, 256, 128, 16.0, False),    # one pair tile per token tile, r = 128
    (1000, 1280, 640, 24, 48.0, False),   # r not a power of two; dX width 640: single CTAs
    (300, 12800, 256, 16, 32.0, True),    # forward: last round split in both shapes
    (300, 256, 12800, 16, 32.0, True),    # dX: the same on the transposed GEMM
])
def test_pair_and_single_against_oracle(q, M, N, K, r, alpha, split):
    p = linear_problem(M, N, K, r, alpha, 0.02, seed=11)
    on, off = _both(q, p)
    TL._check(p, on)
    TL._check(p, off)
    for k, kk in (("Y", K), ("dX", N)):
        d = _apart(on[k], off[k], kk + 2 * r)
        assert d <= (2.0 if split else 0.0), (k, d)
    for k in ("XA", "dA", "dB"):
        assert np.array_equal(on[k], off[k]), k       # not computed by the fused GEMM


@pytest.mark.parametrize("N,K", [(512, 768), (256, 1280)])
def test_pair_dequant_bit_exact_one_hot(q, N, K):
    """X = I and A = 0 make every forward output a single product 1 * w, and dY = I
    every dX output; with pairs on, both GEMMs must reproduce the oracle's
    dequantized bf16 bit for bit, in each CTA's half of the 256-row tile."""
    import torch
    from synth import normal_bf16
    Wb = normal_bf16(0, f"pair_onehot{N}x{K}", (N, K), 0.02)
    ref = H.oracle_deq_bits(Wb)
    prev = q.set_gemm_pairing(True)
    try:
        Wq = q.nf4_quantize(H.bits_to_dev(Wb))
        r = 16
        A = torch.zeros(K, r, dtype=torch.bfloat16, device="cuda")
        B = torch.randn(r, N, device="cuda").to(torch.bfloat16)
        Y, _ = q.linear_fwd(torch.eye(K, dtype=torch.bfloat16, device="cuda"), Wq, A, B, 2.0)
        X0 = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
        dX, _, _ = q.linear_bwd(torch.eye(N, dtype=torch.bfloat16, device="cuda"), X0, None, Wq, A, B, 2.0)
        torch.cuda.synchronize()
    finally:
        q.set_gemm_pairing(prev)
    assert q.device_status() == (0, 0)
    assert np.array_equal(H.dev_to_bits(Y), ref.T)
    assert np.array_equal(H.dev_to_bits(dX), ref)


def test_pairing_switch_keeps_workspace_size(q):
    """Workspace sizes cover either shape: one workspace serves calls made with
    the switch in both positions (a split shape, where the two differ most)."""
    import torch
    p = linear_problem(4096, 4096, 4096, 16, 32.0, 0.02, seed=2)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    ws = q.make_workspace(p.M, p.N, p.K, p.r, X.device)
    prev = q.set_gemm_pairing(True)
    try:
        Y1, XA1 = q.linear_fwd(X, Wq, A, B, p.s, workspace=ws)
        dX1, _, _ = q.linear_bwd(dY, X, XA1, Wq, A, B, p.s, workspace=ws)
        q.set_gemm_pairing(False)
        Y0, XA0 = q.linear_fwd(X, Wq, A, B, p.s, workspace=ws)
        dX0, _, _ = q.linear_bwd(dY, X, XA0, Wq, A, B, p.s, workspace=ws)
        torch.cuda.synchronize()
    finally:
        q.set_gemm_pairing(prev)
    assert q.device_status() == (0, 0)
    assert _apart(H.dev_to_bits(Y1), H.dev_to_bits(Y0), p.K + 2 * p.r) <= 2.0
    assert _apart(H.dev_to_bits(dX1), H.dev_to_bits(dX0), p.N + 2 * p.r) <= 2.0


def test_gemm_units_on_device(q):
    """The single-CTA unit count is the SM count; the pairs the device holds at once
    are between one and half of it."""
    import torch
    ctas, pairs = q.gemm_units()
    assert ctas == torch.cuda.get_device_properties(0).multi_processor_count
    assert 1 <= pairs <= ctas // 2
