"""GPU parity of the merge path (the adapter folded into a 16-bit weight for
serving: "QLoRA", ozercemkelahmet.com, How it works, Step 8 and section "Merging
after QLoRA") against the fp64 oracle (oracle.linear.merge_weight).

The oracle rounds the exact value x = base + s (A B)^T once to bf16.  The kernel
accumulates (A B)^T in fp32 on the tensor cores (r exact products), forms
fma(s, acc, base) in fp32 and rounds that to bf16.  Its fp32 value is within
E = (r + 1) 2^-23 |s| (|A| |B|)^T + 2^-23 |x| of x, so its bf16 result g can
differ from the oracle's only where x lies within E of g's rounding interval:
|x - g| <= E + half a bf16 step at g.  Near a rounding boundary that is one
step; where base and adapter term cancel it can be several (x is then tiny
against the terms, whose fp32 error E stays).  The test checks that condition
for every element that differs, and that such elements stay rare.  With B = 0
the output is the base itself, bit
for bit (for an NF4 base: the standalone dequant's output)."""
import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from synth import linear_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _ordered(bits):
    b = np.asarray(bits, np.uint16).astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _from_ordered(o):
    o = np.asarray(o, np.int64)
    return np.where(o < 0, 0x8000 | (-o), o).astype(np.uint16)


def _rounding_interval(g_bits):
    """The interval of reals that round (nearest) to each bf16 value: halfway to
    its neighbours on either side (asymmetric at a power of two)."""
    o = _ordered(g_bits)
    v = H.onf4.bf16_to_f32(g_bits).astype(np.float64)
    lo = H.onf4.bf16_to_f32(_from_ordered(o - 1)).astype(np.float64)
    hi = H.onf4.bf16_to_f32(_from_ordered(o + 1)).astype(np.float64)
    return 0.5 * (v + lo), 0.5 * (v + hi)


def _check_merge(got, want, Wb, A, B, s, r):
    bad = np.nonzero(got.ravel() != want.ravel())[0]
    if bad.size:
        x = (olin.as_f64(Wb) + s * (olin.as_f64(A) @ olin.as_f64(B)).T).ravel()[bad]
        mag = (np.abs(olin.as_f64(A)) @ np.abs(olin.as_f64(B))).T.ravel()[bad]
        E = (r + 1) * 2.0 ** -23 * abs(s) * mag + 2.0 ** -23 * np.abs(x)
        lo, hi = _rounding_interval(got.ravel()[bad])
        dist = np.maximum(0.0, np.maximum(lo - x, x - hi))   # from x to where the GPU value rounds from
        assert np.all(dist <= E), "a difference not explained by fp32 rounding"
        steps = np.abs(_ordered(got.ravel()[bad]) - _ordered(want.ravel()[bad]))
        far = steps > 1                               # only where base and adapter cancel
        assert np.all(np.abs(x[far]) < 2.0 ** -6 * abs(s) * mag[far] + 1e-30)
    assert bad.size <= max(8, got.size // 2000), (bad.size, got.size)
    return bad.size


@pytest.mark.parametrize("base", ["bf16 original", "dequantized NF4"])
@pytest.mark.parametrize("N,K,r", [(128, 256, 8), (384, 640, 16), (256, 1024, 64), (136, 512, 128),
                                   (4096, 4096, 16), (8192, 8192, 64)])
def test_merge(q, base, N, K, r):
    import torch
    p = linear_problem(1, N, K, r, 2.0 * r, 0.02, seed=N + r, with_dy=False)
    A, B = H.bits_to_dev(p.A), H.bits_to_dev(p.B)
    s = 2.0
    if base == "bf16 original":
        Wb = p.W
        out = q.nf4_merge(A, B, s, W16=H.bits_to_dev(p.W))
    else:
        Wb = H.oracle_deq_bits(p.W)
        out = q.nf4_merge(A, B, s, Wq=q.nf4_quantize(H.bits_to_dev(p.W)))
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    got = H.dev_to_bits(out)
    want = olin.merge_weight(Wb, p.A, p.B, s)
    _check_merge(got, want, Wb, p.A, p.B, s, r)


def test_merge_large_adapter_many_ties(q):
    """B ~ N(0, 1) makes the adapter term as large as the weights, so many more
    elements land near a rounding boundary; each difference must still be one
    explained by fp32 rounding."""
    import torch
    from synth import normal_bf16
    N, K, r = 512, 1024, 32
    p = linear_problem(1, N, K, r, 2.0 * r, 0.02, seed=9, with_dy=False)
    Bb = normal_bf16(9, "Bbig", (r, N), 1.0)
    out = q.nf4_merge(H.bits_to_dev(p.A), H.bits_to_dev(Bb), 0.5, W16=H.bits_to_dev(p.W))
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    want = olin.merge_weight(p.W, p.A, Bb, 0.5)
    _check_merge(H.dev_to_bits(out), want, p.W, p.A, Bb, 0.5, r)


@pytest.mark.parametrize("base", ["bf16 original", "dequantized NF4"])
def test_merge_without_adapter_is_the_base(q, base):
    import torch
    p = linear_problem(1, 256, 512, 16, 32.0, 0.02, seed=5, with_dy=False)
    A = H.bits_to_dev(p.A)
    B = torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda")
    if base == "bf16 original":
        W16 = H.bits_to_dev(p.W)
        out = q.nf4_merge(A, B, 2.0, W16=W16)
        ref = W16
    else:
        Wq = q.nf4_quantize(H.bits_to_dev(p.W))
        out = q.nf4_merge(A, B, 2.0, Wq=Wq)
        ref = q.nf4_dequant(Wq)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_merge_argument_errors(q):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    A = torch.zeros(128, 16, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    W16 = torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda")
    Wq = q.nf4_quantize(W16)
    with pytest.raises(ValueError):
        q.nf4_merge(A, B, 1.0)                              # no base
    with pytest.raises(ValueError):
        q.nf4_merge(A, B, 1.0, Wq=Wq, W16=W16)              # two bases
    with pytest.raises(_abi.QloraError):
        q.nf4_merge(torch.zeros(128, 12, dtype=torch.bfloat16, device="cuda"),
                    torch.zeros(12, 128, dtype=torch.bfloat16, device="cuda"), 1.0, W16=W16)   # r % 8
