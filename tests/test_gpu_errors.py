"""GPU error paths: bounded device waits report a timeout instead of hanging, the
context stays usable afterwards, and argument errors are returned before any
launch.  No test traps, faults or hangs the GPU."""
import numpy as np
import pytest

import helpers as H
from synth import normal_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def test_wait_timeout_is_reported_and_context_survives(q):
    import torch
    assert q.device_status()[0] == 0
    assert q.selftest_wait_timeout(2000) == 0          # 2 ms on a barrier nobody arrives on
    code, flags = q.device_status()
    assert code == 5 and (flags & 1)
    assert q.device_status() == (0, 0)                  # cleared
    bits = normal_bf16(0, "after-timeout", (64, 128), 0.02)
    Wq = q.nf4_quantize(H.bits_to_dev(bits, (64, 128)))
    torch.cuda.synchronize()
    ref = H.oracle_quantize_bits(bits.ravel())
    assert np.array_equal(Wq.codes.cpu().numpy(), ref["codes"])


def test_workspace_errors(q):
    import torch
    from bit_nf4_quantized_19_b200 import _abi
    X = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    Wq = q.nf4_quantize(torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda"))
    A = torch.zeros(256, 8, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(_abi.QloraError) as e:
        q.linear_fwd(X, Wq, A, B, 1.0, workspace=small)
    assert e.value.code == 7
    with pytest.raises(ValueError):
        q.linear_fwd(X[:, 1:], Wq, A, B, 1.0)          # K does not match the weight
