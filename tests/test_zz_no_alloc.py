"""The forward without a workspace argument (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory: a host program that links
only this library and has no device allocator, or a runtime that plans all device
memory up front and forbids allocations while it runs.  Its scratch lives in one
fixed device array inside the library, shared by every call on a device.

Checked here through the C ABI, against the fp64 oracle with the bars of the
linear tests (Y within one bf16 ulp element-wise and 2e-3 relative Frobenius; XA
within 2^-15 of |X| |A| and 1e-4):
  - the large-token path at a shape whose GEMM splits its last round (4096 tokens
    on a 4096 x 4096 weight): partial tiles and their arrival counters live in the
    fixed array, and whatever the array held before must not leak in;
  - the few-token path with XA_out = NULL (M = 1 and 16), where XA itself lives in
    the fixed array;
  - every case twice in a row with different inputs, so stale scratch from the
    first call would show in the second;
  - a call needing more scratch than the array holds is rejected before any launch.
Collected last, so that a run stopping at the first failure has run everything
else first."""
import ctypes

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


def _noalloc_fwd(X, Wq, A, B, s, want_xa):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    M, r = X.shape[0], A.shape[1]
    Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=X.device)
    XA = torch.empty(M, r, dtype=torch.float32, device=X.device) if want_xa else None
    st = Wq.c_struct()
    code = _abi.lib().qlora_linear_fwd_noalloc(
        ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(st), ctypes.c_void_p(A.data_ptr()),
        ctypes.c_void_p(B.data_ptr()), r, float(s), ctypes.c_void_p(Y.data_ptr()),
        ctypes.c_void_p(XA.data_ptr()) if want_xa else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return code, Y, XA


@pytest.mark.parametrize("M,N,K,r,want_xa,rows", [
    (4096, 4096, 4096, 16, False, 64),   # GEMM with a split last round; scratch ~9 MB
    (4096, 4096, 4096, 16, True, 64),
    (300, 384, 512, 16, True, None),
    (1, 4096, 4096, 16, False, None),    # few-token path, XA only in the fixed array
    (16, 11008, 4096, 16, False, None),
])
def test_noalloc_forward_matches_oracle_twice(q, M, N, K, r, want_xa, rows):
    import torch
    p0 = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=41, with_dy=False)
    Wd = H.oracle_deq_bits(p0.W)
    Wq = q.nf4_quantize(H.bits_to_dev(p0.W))
    A, B = H.bits_to_dev(p0.A), H.bits_to_dev(p0.B)
    sel = None
    if rows is not None:
        sel = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(7).integers(0, M, rows)]))
    for call, seed in enumerate((42, 43)):
        p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=seed, with_dy=False)
        code, Y, XA = _noalloc_fwd(H.bits_to_dev(p.X), Wq, A, B, p0.s, want_xa)
        assert code == 0, f"call {call}: status {code}"
        torch.cuda.synchronize()
        assert q.device_status() == (0, 0)
        Yb = H.dev_to_bits(Y)
        X = p.X if sel is None else p.X[sel]
        Yref, XAref = olin.forward(X, Wd, p0.A, p0.B, p0.s)
        Yg = Yb if sel is None else Yb[sel]
        assert olin.rel_fro(H.onf4.bf16_to_f32(Yg), Yref) <= TOL_BF16, call
        assert H.bf16_ulp_check(Yg, Yref, K + 2 * r) <= 1.0, call
        if want_xa:
            xa = XA.cpu().numpy().astype(np.float64)
            xa = xa if sel is None else xa[sel]
            assert olin.rel_fro(xa, XAref) <= TOL_FP32, call
            mag = np.abs(olin.as_f64(X)) @ np.abs(olin.as_f64(p0.A))
            assert H.mag_check(xa, XAref, mag) <= 1.0, call


def test_noalloc_rejects_oversized_call_before_launch(q):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    Wq = q.nf4_quantize(torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda"))
    X = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(128, 16, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(8, 128, dtype=torch.bfloat16, device="cuda")
    st = Wq.c_struct()
    huge_m = 1 << 22          # needs far more than the library's fixed scratch array
    code = _abi.lib().qlora_linear_fwd_noalloc(
        ctypes.c_void_p(X.data_ptr()), huge_m, ctypes.byref(st), ctypes.c_void_p(A.data_ptr()),
        ctypes.c_void_p(B.data_ptr()), 16, 1.0, ctypes.c_void_p(Y.data_ptr()), None, None)
    assert code == _abi.QLORA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert q.device_status() == (0, 0)
