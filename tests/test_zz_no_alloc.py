"""The forward without a workspace argument (qlora_linear_fwd_noalloc), for callers
that cannot allocate device memory -- e.g. a host program that links only this
library and has no device allocator, or a runtime that plans all device memory
up front and forbids allocations at call time.  Its scratch lives in a fixed
device array inside the library.

Checked here through the C ABI: two calls in a row (different inputs, so stale
scratch from the first call would show in the second) each match the regular
forward (which takes a caller workspace) within the tolerances of the linear
tests; a call needing more scratch than the array holds is rejected before any
launch.  Collected last so that a first-failure stop has run everything else."""
import ctypes

import numpy as np
import pytest

import helpers as H
from oracle import linear as olin
from synth import linear_problem

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_FP32 = 1e-4


def _noalloc_fwd(q, X, Wq, A, B, s):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    M, r = X.shape[0], A.shape[1]
    Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=X.device)
    XA = torch.empty(M, r, dtype=torch.float32, device=X.device)
    st = Wq.c_struct()
    code = _abi.lib().qlora_linear_fwd_noalloc(
        ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(st), ctypes.c_void_p(A.data_ptr()),
        ctypes.c_void_p(B.data_ptr()), r, float(s), ctypes.c_void_p(Y.data_ptr()),
        ctypes.c_void_p(XA.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return code, Y, XA


def test_noalloc_forward_matches_workspace_forward_twice():
    import torch
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    for call, (M, N, K, r, seed) in enumerate([(300, 384, 512, 16, 11), (1000, 512, 256, 24, 12)]):
        p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=seed)
        X, A, B = H.bits_to_dev(p.X), H.bits_to_dev(p.A), H.bits_to_dev(p.B)
        Wq = q.nf4_quantize(H.bits_to_dev(p.W))
        Y_ref, XA_ref = q.linear_fwd(X, Wq, A, B, p.s)
        code, Y, XA = _noalloc_fwd(q, X, Wq, A, B, p.s)
        assert code == 0, f"call {call}: status {code}"
        torch.cuda.synchronize()
        assert q.device_status() == (0, 0)
        yr = H.onf4.bf16_to_f32(H.dev_to_bits(Y_ref)).astype(np.float64)
        yn = H.onf4.bf16_to_f32(H.dev_to_bits(Y)).astype(np.float64)
        assert olin.rel_fro(yn, yr) <= TOL_BF16, call
        assert olin.rel_fro(XA.cpu().numpy(), XA_ref.cpu().numpy()) <= TOL_FP32, call


def test_noalloc_rejects_oversized_call_before_launch():
    import torch
    import bit_nf4_quantized_19_b200 as q
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
