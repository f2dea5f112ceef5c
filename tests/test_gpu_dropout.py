"""GPU parity of the LoRA extras against the fp64 oracle: dropout on the adapter
input ("QLoRA", ozercemkelahmet.com, "A code example with common libraries":
lora_dropout; oracle.linear.forward_dropout / backward_dropout) and gradient
accumulation over micro-batches ("Training arguments":
gradient_accumulation_steps; oracle.linear.accumulate_grads).

The keep mask is an input drawn on the host (synth.keep_mask) and handed to the
library bit-packed.  Bars as in test_gpu_linear: Y and dX within 2e-3 relative
Frobenius and one bf16 ulp element-wise; XA, dA and dB within 1e-4 and 2^-15 of
their magnitude products (here over the dropped-out input X (.) keep / (1-p))."""
import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from synth import keep_mask, linear_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _bits(keep):
    return np.packbits(keep.astype(np.uint8).ravel(), bitorder="little")


def _dev_bits(keep):
    import torch
    return torch.from_numpy(_bits(keep)).cuda()


def _check(p, keep, pdrop, Yb, XA, dXb, dA, dB, XA_in_bwd=None):
    Wd = H.oracle_deq_bits(p.W)
    Y, XAr = olin.forward_dropout(p.X, Wd, p.A, p.B, p.s, keep, pdrop)
    g = olin.backward_dropout(p.dY, p.X, Wd, p.A, p.B, p.s, keep, pdrop)
    assert olin.rel_fro(H.onf4.bf16_to_f32(Yb), Y) <= 2e-3
    assert H.bf16_ulp_check(Yb, Y, p.K + 2 * p.r) <= 1.0
    if dXb is not None:
        assert olin.rel_fro(H.onf4.bf16_to_f32(dXb), g["dX"]) <= 2e-3
        assert H.bf16_ulp_check(dXb, g["dX"], p.N + 2 * p.r) <= 1.0
    Xd = olin.dropout_input(p.X, keep, pdrop)
    mag = H.lora_magnitudes(Xd, p.A, p.B, p.dY, p.s, XA=XAr)
    for name, got, ref in (("XA", XA, XAr), ("dA", dA, g["dA"]), ("dB", dB, g["dB"])):
        if got is None:
            continue
        assert olin.rel_fro(got, ref) <= 1e-4, name
        assert H.mag_check(got, ref, mag[name]) <= 1.0, name


@pytest.mark.parametrize("M,N,K,r,pdrop", [
    (300, 384, 256, 16, 0.05),
    (513, 256, 384, 64, 0.5),
    (300, 256, 12800, 16, 0.1),     # dX GEMM with its last round split in contraction halves
    (300, 12800, 256, 16, 0.1),     # forward GEMM split
    (16, 1024, 1024, 8, 0.05),      # few-token forward, large-M backward
    (1, 256, 512, 16, 0.3),
])
@pytest.mark.parametrize("saved_xa", [True, False])
def test_dropout_fwd_bwd(q, M, N, K, r, pdrop, saved_xa):
    import torch
    p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=M + N)
    keep = keep_mask(M, f"{M}x{N}x{K}", (M, K), pdrop)
    kb = _dev_bits(keep)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    Y, XA = q.linear_fwd(X, Wq, A, B, p.s, keep_bits=kb, dropout_p=pdrop)
    dX, dA, dB = q.linear_bwd(dY, X, XA if saved_xa else None, Wq, A, B, p.s, keep_bits=kb, dropout_p=pdrop)
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    _check(p, keep, pdrop, H.dev_to_bits(Y), XA.cpu().numpy().astype(np.float64), H.dev_to_bits(dX),
           dA.cpu().numpy().astype(np.float64), dB.cpu().numpy().astype(np.float64))


def test_everything_dropped(q):
    """keep = 0 everywhere: XA = 0, dA = 0, and Y, dX are the frozen path alone."""
    import torch
    M, N, K, r = 300, 384, 256, 16
    p = linear_problem(M, N, K, r, 32.0, 0.02, seed=4)
    keep = np.zeros((M, K), bool)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    Y, XA = q.linear_fwd(X, Wq, A, B, p.s, keep_bits=_dev_bits(keep), dropout_p=0.25)
    dX, dA, dB = q.linear_bwd(dY, X, XA, Wq, A, B, p.s, keep_bits=_dev_bits(keep), dropout_p=0.25)
    torch.cuda.synchronize()
    assert float(XA.abs().max()) == 0.0 and float(dA.abs().max()) == 0.0 and float(dB.abs().max()) == 0.0
    _check(p, keep, 0.25, H.dev_to_bits(Y), None, H.dev_to_bits(dX), None, None)


@pytest.mark.parametrize("dropout", [False, True])
def test_gradient_accumulation(q, dropout):
    """Three micro-batches: the first backward overwrites dA and dB, the next two add
    into them; the sum equals the oracle's accumulated gradients."""
    import torch
    N, K, r = 384, 512, 16
    acc = None
    dA = torch.full((K, r), float("nan"), dtype=torch.float32, device="cuda")
    dB = torch.full((r, N), float("nan"), dtype=torch.float32, device="cuda")
    mags = None
    from synth import normal_bf16
    base = linear_problem(1, N, K, r, 32.0, 0.02, seed=70)     # one W, A, B for every micro-batch
    for i, M in enumerate((200, 300, 17)):
        p = linear_problem(1, N, K, r, 32.0, 0.02, seed=70)
        p.M = M
        p.X = normal_bf16(i, "accX", (M, K), 1.0)
        p.dY = normal_bf16(i, "accdY", (M, N), 1.0)
        assert np.array_equal(p.W, base.W) and np.array_equal(p.A, base.A)
        keep = keep_mask(i, "acc", (M, K), 0.1) if dropout else np.ones((M, K), bool)
        kb = _dev_bits(keep) if dropout else None
        X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
        Wq = q.nf4_quantize(H.bits_to_dev(p.W))
        Y, XA = q.linear_fwd(X, Wq, A, B, p.s, keep_bits=kb, dropout_p=0.1 if dropout else 0.0)
        q.linear_bwd(dY, X, XA, Wq, A, B, p.s, need_dx=False, dA=dA, dB=dB, keep_bits=kb,
                     dropout_p=0.1 if dropout else 0.0, accumulate=i > 0)
        Wd = H.oracle_deq_bits(p.W)
        g = olin.backward_dropout(p.dY, p.X, Wd, p.A, p.B, p.s, keep, 0.1 if dropout else 0.0)
        acc = olin.accumulate_grads(acc, g)
        Xd = olin.dropout_input(p.X, keep, 0.1 if dropout else 0.0)
        XAr = Xd @ olin.as_f64(p.A)
        m = H.lora_magnitudes(Xd, p.A, p.B, p.dY, p.s, XA=XAr)
        mags = m if mags is None else {k: mags[k] + m[k] for k in ("dA", "dB")}
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    for name, got in (("dA", dA), ("dB", dB)):
        got = got.cpu().numpy().astype(np.float64)
        assert olin.rel_fro(got, acc[name]) <= 1e-4, name
        assert H.mag_check(got, acc[name], mags[name]) <= 1.0, name


def test_dropout_argument_errors(q):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    X = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    Wq = q.nf4_quantize(torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda"))
    A = torch.zeros(128, 16, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros(8 * 128 // 8, dtype=torch.uint8, device="cuda")
    for bad_p in (1.0, -0.1, float("nan")):
        with pytest.raises(_abi.QloraError):
            q.linear_fwd(X, Wq, A, B, 1.0, keep_bits=kb, dropout_p=bad_p)
    with pytest.raises(_abi.QloraError):     # a plain-size workspace has no room for X (.) keep
        q.linear_fwd(X, Wq, A, B, 1.0, keep_bits=kb, dropout_p=0.1,
                     workspace=q.make_workspace(8, 128, 128, 16, X.device))
