"""GPU parity of the fused QLoRA linear forward and backward against the fp64
oracle over the same dequantized weights.

Bar (per output): ||gpu - oracle||_F / ||oracle||_F <= 2e-3 for Y and dX (bf16
outputs; bf16 rounding alone costs ~1.66e-3), and <= 1e-4 for the fp32
outputs XA, dA and dB (fp32 accumulation over at most 8192 tokens; a bf16
intermediate anywhere in those paths would show up as ~1e-3).  Y and dX are
also checked element-wise: within one bf16 ulp of the exact value, with an
absolute floor of 4 sqrt(K) 2^-23 rms for results that cancel to near zero.
XA, dA and dB are checked element-wise too: within 2^-15 of the product of the
operands' magnitudes (helpers.mag_check)."""
import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from synth import linear_problem

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_FP32 = 1e-4


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _run(q, p, rows=None, xa_to_bwd=True, need_dx=True):
    import torch
    X = H.bits_to_dev(p.X)
    A = H.bits_to_dev(p.A)
    B = H.bits_to_dev(p.B)
    dY = H.bits_to_dev(p.dY)
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    ws = q.make_workspace(p.M, p.N, p.K, p.r, X.device)
    Y, XA = q.linear_fwd(X, Wq, A, B, p.s, workspace=ws)
    dX, dA, dB = q.linear_bwd(dY, X, XA if xa_to_bwd else None, Wq, A, B, p.s,
                              need_dx=need_dx, workspace=ws)
    torch.cuda.synchronize()
    code, flags = q.device_status()
    assert code == 0 and flags == 0
    out = dict(Y=H.dev_to_bits(Y), XA=XA.cpu().numpy().astype(np.float64),
               dA=dA.cpu().numpy().astype(np.float64), dB=dB.cpu().numpy().astype(np.float64))
    if dX is not None:
        out["dX"] = H.dev_to_bits(dX)
    return out


def _check(p, got, rows=None):
    Wd = H.oracle_deq_bits(p.W)
    if rows is None:
        Y, XA = olin.forward(p.X, Wd, p.A, p.B, p.s)
        g = olin.backward(p.dY, p.X, Wd, p.A, p.B, p.s)
        Yg, dXg = got["Y"], got.get("dX")
    else:
        Y, _ = olin.forward_rows(p.X, Wd, p.A, p.B, p.s, rows)
        g = olin.lora_products(p.dY, p.X, p.A, p.B, p.s)     # XA, dA, dB need no W
        XA = g["XA"]
        g["dX"] = olin.backward_rows_dx(p.dY, Wd, p.A, p.B, p.s, rows)
        Yg = got["Y"][rows]
        dXg = got["dX"][rows] if "dX" in got else None
    errs = {
        "Y": olin.rel_fro(H.onf4.bf16_to_f32(Yg), Y),
        "XA": olin.rel_fro(got["XA"], XA),
        "dA": olin.rel_fro(got["dA"], g["dA"]),
        "dB": olin.rel_fro(got["dB"], g["dB"]),
    }
    assert errs["Y"] <= TOL_BF16, errs
    assert H.bf16_ulp_check(Yg, Y, p.K + 2 * p.r) <= 1.0, errs
    assert errs["XA"] <= TOL_FP32 and errs["dA"] <= TOL_FP32 and errs["dB"] <= TOL_FP32, errs
    mag = H.lora_magnitudes(p.X, p.A, p.B, p.dY, p.s, XA=XA)
    for k in ("XA", "dA", "dB"):
        ref = XA if k == "XA" else g[k]
        errs[k + "_mag"] = H.mag_check(got[k], ref, mag[k])
        assert errs[k + "_mag"] <= 1.0, (k, errs)
    if dXg is not None:
        errs["dX"] = olin.rel_fro(H.onf4.bf16_to_f32(dXg), g["dX"])
        assert errs["dX"] <= TOL_BF16, errs
        assert H.bf16_ulp_check(dXg, g["dX"], p.N + 2 * p.r) <= 1.0, errs
    return errs


# small workload of the pages' scale plus shapes that span several tiles and a ragged tail
@pytest.mark.parametrize("M,N,K,r,alpha", [
    (16, 1024, 1024, 8, 16.0),     # the small single-layer workload
    (1, 256, 512, 16, 32.0),
    (4, 256, 512, 16, 32.0),
    (17, 384, 256, 8, 16.0),
    (300, 384, 256, 16, 32.0),     # 2 token tiles (ragged), 3 weight tiles
    (513, 256, 384, 64, 16.0),     # r=64: two LoRA stages
    (257, 128, 256, 128, 16.0),    # r=128: four LoRA stages
    (1000, 640, 896, 24, 48.0),    # r not a power of two
    (300, 12800, 256, 16, 32.0),   # forward: 200 tiles on 148 CTAs, last round split in contraction halves
    (300, 256, 12800, 16, 32.0),   # dX: the same split on the transposed GEMM
])
def test_linear_fwd_bwd_full(q, M, N, K, r, alpha):
    p = linear_problem(M, N, K, r, alpha, 0.02, seed=0)
    got = _run(q, p)
    _check(p, got)


def test_linear_bwd_without_saved_xa_and_without_dx(q):
    p = linear_problem(200, 256, 384, 16, 32.0, 0.02, seed=1)
    got = _run(q, p, xa_to_bwd=False)
    _check(p, got)
    got2 = _run(q, p, need_dx=False)
    assert "dX" not in got2
    _check(p, got2)


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_linear_llama7b_shapes_sampled_rows(q, N, K):
    """The 4096-token LLaMA-7B-shaped projections at full size, in the launch
    configuration the bench times; Y and dX checked on 96 seeded token rows
    (including the first and last), XA, dA and dB in full."""
    p = linear_problem(4096, N, K, 16, 32.0, 0.02, seed=0)
    got = _run(q, p)
    rows = np.unique(np.concatenate([[0, 4095], np.random.default_rng(5).integers(0, 4096, 94)]))
    _check(p, got, rows=rows)


@pytest.mark.parametrize("N,K", [(8192, 8192), (22016, 8192), (8192, 22016)])
def test_linear_llama65b_shapes_sampled_rows(q, N, K):
    """The 8192-token LLaMA-65B-shaped projections (r = 64, alpha = 16, W ~ N(0, 0.015))
    at full size; Y and dX on 48 seeded token rows (including the first and last),
    XA, dA and dB in full."""
    p = linear_problem(8192, N, K, 64, 16.0, 0.015, seed=0)
    got = _run(q, p)
    rows = np.unique(np.concatenate([[0, 8191], np.random.default_rng(6).integers(0, 8192, 46)]))
    _check(p, got, rows=rows)


@pytest.mark.parametrize("M,N,K,r", [(384, 256, 384, 16), (256, 640, 256, 64)])
def test_projection_G_direct(q, M, N, K, r):
    """G = dY B^T checked on its own: with X = the first K rows of the identity
    (M = K tokens, the rest zero), dA = s X^T G is s G[k, :] for k < K, carried
    through the gradient kernel as bf16 hi + lo, i.e. to 2^-17 relative.  So
    every element of s G is compared with the oracle's, within 2^-15 of its
    magnitude product s |dY| |B|^T."""
    import torch
    p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=21)
    Xi = np.zeros((M, K), np.uint16)
    Xi[np.arange(min(M, K)), np.arange(min(M, K))] = 0x3F80          # bf16 1.0
    X = H.bits_to_dev(Xi)
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    A, B, dY = H.bits_to_dev(p.A), H.bits_to_dev(p.B), H.bits_to_dev(p.dY)
    _, dA, _ = q.linear_bwd(dY, X, None, Wq, A, B, p.s, need_dx=False)
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    G = olin.as_f64(p.dY) @ olin.as_f64(p.B).T
    n = min(M, K)
    got = dA.cpu().numpy().astype(np.float64)[:n]
    mag = abs(p.s) * (np.abs(olin.as_f64(p.dY)) @ np.abs(olin.as_f64(p.B)).T)[:n]
    assert H.mag_check(got, p.s * G[:n], mag) <= 1.0


@pytest.mark.parametrize("N,K", [(256, 384), (384, 256), (128, 1024)])
def test_gemm_dequant_bit_exact_one_hot(q, N, K):
    """With X = I (K one-hot tokens) and A = 0 every output of the forward is a
    single product 1 * w, so Y = deq(W)^T exactly; with dY = I (N tokens),
    dX = deq(W).  The dequantization inside both fused GEMMs must therefore
    equal the oracle's dequantized bf16 bit for bit."""
    import torch
    from synth import normal_bf16
    Wb = normal_bf16(0, f"onehot{N}x{K}", (N, K), 0.02)
    ref = H.oracle_deq_bits(Wb)                                   # [N, K] bf16 bits
    Wq = q.nf4_quantize(H.bits_to_dev(Wb))
    r = 16
    A = torch.zeros(K, r, dtype=torch.bfloat16, device="cuda")
    B = torch.randn(r, N, device="cuda").to(torch.bfloat16)
    Xi = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    Y, _ = q.linear_fwd(Xi, Wq, A, B, 2.0)
    dYi = torch.eye(N, dtype=torch.bfloat16, device="cuda")
    X0 = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    dX, _, _ = q.linear_bwd(dYi, X0, None, Wq, A, B, 2.0)
    torch.cuda.synchronize()
    assert np.array_equal(H.dev_to_bits(Y), ref.T)
    assert np.array_equal(H.dev_to_bits(dX), ref)


def test_fwd_bwd_capture_in_cuda_graph(q):
    """The forward and backward capture into one CUDA graph; replays give
    bit-identical results to eager calls."""
    import torch
    p = linear_problem(64, 384, 512, 16, 32.0, 0.02, seed=3)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    ws = q.make_workspace(p.M, p.N, p.K, p.r, X.device)
    Y = torch.empty(p.M, p.N, dtype=torch.bfloat16, device="cuda")
    XA = torch.empty(p.M, p.r, dtype=torch.float32, device="cuda")
    dX = torch.empty(p.M, p.K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(p.K, p.r, dtype=torch.float32, device="cuda")
    dB = torch.empty(p.r, p.N, dtype=torch.float32, device="cuda")

    def step():
        q.linear_fwd(X, Wq, A, B, p.s, workspace=ws, Y=Y, XA=XA)
        q.linear_bwd(dY, X, XA, Wq, A, B, p.s, workspace=ws, dX=dX, dA=dA, dB=dB)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (Y, XA, dX, dA, dB)]
    for t in (Y, XA, dX, dA, dB):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    for got, want in zip((Y, XA, dX, dA, dB), ref):
        assert torch.equal(got.view(torch.int16) if got.dtype == torch.bfloat16 else got.view(torch.int32),
                           want.view(torch.int16) if want.dtype == torch.bfloat16 else want.view(torch.int32))


def test_graph_replay_with_new_inputs_at_a_split_shape(q):
    """4096 tokens on a 4096 x 4096 weight make 512 GEMM tiles on 148 SMs: the 68
    tiles of the last round are split in contraction halves in both the forward
    and the dX GEMM.  A forward + backward captured once and replayed with new X
    and dY in the same buffers must give, bit for bit, what eager calls give on
    those inputs (the split tiles' arrival counters must start from zero on every
    replay)."""
    import torch
    M, N, K, r = 4096, 4096, 4096, 16
    ps = [linear_problem(M, N, K, r, 32.0, 0.02, seed=sd) for sd in (31, 32, 33)]
    Wq = q.nf4_quantize(H.bits_to_dev(ps[0].W))
    A, B = H.bits_to_dev(ps[0].A), H.bits_to_dev(ps[0].B)
    X = H.bits_to_dev(ps[0].X)
    dY = H.bits_to_dev(ps[0].dY)
    ws = q.make_workspace(M, N, K, r, X.device)
    outs = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda"),
            torch.empty(M, r, dtype=torch.float32, device="cuda"),
            torch.empty(M, K, dtype=torch.bfloat16, device="cuda"),
            torch.empty(K, r, dtype=torch.float32, device="cuda"),
            torch.empty(r, N, dtype=torch.float32, device="cuda")]
    s = ps[0].s

    def step(Xt, dYt, Y, XA, dX, dA, dB):
        q.linear_fwd(Xt, Wq, A, B, s, workspace=ws, Y=Y, XA=XA)
        q.linear_bwd(dYt, Xt, XA, Wq, A, B, s, workspace=ws, dX=dX, dA=dA, dB=dB)

    step(X, dY, *outs)                                  # eager warm-up on the first inputs
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(X, dY, *outs)
    for p in ps[1:]:
        X.copy_(H.bits_to_dev(p.X))
        dY.copy_(H.bits_to_dev(p.dY))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in outs]
        ref = [torch.empty_like(t) for t in outs]
        step(X, dY, *ref)
        torch.cuda.synchronize()
        assert q.device_status() == (0, 0)
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))
    del g


@pytest.mark.gpu
def test_capture_before_any_eager_call(q):
    """A shape whose launch geometry the library has not chosen yet (the cluster
    occupancy is queried on first use) captures into a CUDA graph as its first call;
    replays match a later eager call bit for bit."""
    import torch
    p = linear_problem(200, 640, 768, 24, 48.0, 0.02, seed=11)
    X, A, B, dY = (H.bits_to_dev(v) for v in (p.X, p.A, p.B, p.dY))
    Wq = q.nf4_quantize(H.bits_to_dev(p.W))
    ws = q.make_workspace(p.M, p.N, p.K, p.r, X.device)
    outs = [torch.empty(p.M, p.N, dtype=torch.bfloat16, device="cuda"),
            torch.empty(p.M, p.r, dtype=torch.float32, device="cuda"),
            torch.empty(p.M, p.K, dtype=torch.bfloat16, device="cuda"),
            torch.empty(p.K, p.r, dtype=torch.float32, device="cuda"),
            torch.empty(p.r, p.N, dtype=torch.float32, device="cuda")]

    def step(Y, XA, dX, dA, dB):
        q.linear_fwd(X, Wq, A, B, p.s, workspace=ws, Y=Y, XA=XA)
        q.linear_bwd(dY, X, XA, Wq, A, B, p.s, workspace=ws, dX=dX, dA=dA, dB=dB)

    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(*outs)
    g.replay()
    torch.cuda.synchronize()
    ref = [torch.empty_like(t) for t in outs]
    step(*ref)
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
    for got, want in zip(outs, ref):
        assert torch.equal(got.view(torch.int16) if got.dtype == torch.bfloat16 else got.view(torch.int32),
                           want.view(torch.int16) if want.dtype == torch.bfloat16 else want.view(torch.int32))


@pytest.mark.parametrize("N,K", [(22016, 8192), (4096, 4096)])
def test_full_output_repeated_against_fp32_gemm(q, N, K):
    """Every element of Y and dX, over five repeated calls, against an fp32 cuBLAS
    product (TF32 off) of the same bf16 operands and the library's dequantized weight
    (whose bits the tests above pin to the oracle).  The oracle checks sample rows at
    this size; this check covers every tile of every call, so a pipeline race that
    corrupts one tile now and then cannot hide.  Bound per element: one bf16 ulp of
    the reference plus the fp32 accumulation floor of helpers.bf16_ulp_check."""
    import torch
    tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        _full_output_check(q, N, K)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = tf32


def _full_output_check(q, N, K):
    import torch
    M, r = (8192, 64) if N > 8192 else (4096, 16)
    g = torch.Generator(device="cuda")
    g.manual_seed(17)
    W = (torch.randn(N, K, generator=g, device="cuda") * 0.015).to(torch.bfloat16)
    X = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    dY = torch.randn(M, N, generator=g, device="cuda").to(torch.bfloat16)
    A = (torch.randn(K, r, generator=g, device="cuda") / r).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    s = 0.25
    Wq = q.nf4_quantize(W)
    Wd = q.nf4_dequant(Wq).float()
    del W
    Xf, Af, Bf, dYf = X.float(), A.float(), B.float(), dY.float()
    Yref = Xf @ Wd.T + s * ((Xf @ Af) @ Bf)
    dXref = dYf @ Wd + s * ((dYf @ Bf.T) @ Af.T)
    del Xf, dYf

    def bound(ref, contraction):
        mag = ref.abs()
        ulp = torch.exp2(torch.floor(torch.log2(mag.clamp_min(1e-38))) - 7)
        rms = float(ref.square().mean().sqrt())
        return ulp + 4.0 * (contraction ** 0.5) * 2.0 ** -23 * rms

    by, bdx = bound(Yref, K + 2 * r), bound(dXref, N + 2 * r)
    ws = q.make_workspace(M, N, K, r, X.device)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    XA = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    for call in range(5):
        q.linear_fwd(X, Wq, A, B, s, workspace=ws, Y=Y, XA=XA)
        q.linear_bwd(dY, X, XA, Wq, A, B, s, workspace=ws, dX=dX)
        torch.cuda.synchronize()
        assert q.device_status() == (0, 0)
        ey = ((Y.float() - Yref).abs() > by).sum().item()
        edx = ((dX.float() - dXref).abs() > bdx).sum().item()
        assert ey == 0 and edx == 0, (call, ey, edx)
