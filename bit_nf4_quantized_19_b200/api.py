"""Tensor-level wrappers over the C ABI (PyTorch supplies device memory and streams).

Each function allocates its outputs with torch, passes raw device pointers and
the current CUDA stream to libqlora_nf4.so and returns the tensors.  No
arithmetic of the method happens here.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional, Tuple

import torch

from . import _abi


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _bf16_2d(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_cuda:
        raise TypeError(f"{name} must be a 2-D bfloat16 CUDA tensor")
    return t.contiguous()


@dataclasses.dataclass
class NF4Weight:
    """A quantized frozen weight [rows, cols]: packed codes, 8-bit block
    constants, fp32 group constants (device tensors owned by this object).  With
    q8 = None the constants are single-level: `step` holds one fp32 absmax per
    64-value block."""
    codes: torch.Tensor
    q8: Optional[torch.Tensor]
    step: torch.Tensor
    rows: int
    cols: int

    def c_struct(self) -> _abi.NF4Struct:
        return _abi.NF4Struct(self.codes.data_ptr(), self.q8.data_ptr() if self.q8 is not None else None,
                              self.step.data_ptr(), self.rows, self.cols)

    @property
    def single_level(self) -> bool:
        return self.q8 is None

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + (self.q8.numel() if self.q8 is not None else 0) + 4 * self.step.numel()


def nf4_levels() -> list:
    buf = (ctypes.c_float * 16)()
    _abi.lib().qlora_nf4_levels(buf)
    return list(buf)


def nf4_bytes(rows: int, cols: int) -> Tuple[int, int, int]:
    c, q, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _abi.lib().qlora_nf4_bytes(rows, cols, ctypes.byref(c), ctypes.byref(q), ctypes.byref(s))
    return c.value, q.value, s.value


def nf4_empty(rows: int, cols: int, device) -> NF4Weight:
    cb, qb, sb = nf4_bytes(rows, cols)
    return NF4Weight(torch.empty(cb, dtype=torch.uint8, device=device),
                     torch.empty(qb, dtype=torch.uint8, device=device),
                     torch.empty(sb // 4, dtype=torch.float32, device=device), rows, cols)


def nf4_empty_single(rows: int, cols: int, device) -> NF4Weight:
    """Storage for single-level constants (one fp32 absmax per 64-value block)."""
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    _abi.lib().qlora_nf4_single_bytes(rows, cols, ctypes.byref(c), ctypes.byref(s))
    return NF4Weight(torch.empty(c.value, dtype=torch.uint8, device=device), None,
                     torch.empty(s.value // 4, dtype=torch.float32, device=device), rows, cols)


def nf4_quantize(W: torch.Tensor, out: Optional[NF4Weight] = None, single_level: bool = False) -> NF4Weight:
    """Blockwise NF4 quantization of a bf16 [rows, cols] CUDA tensor, with
    double-quantized constants (default) or single-level fp32 ones."""
    W = _bf16_2d(W, "W")
    rows, cols = W.shape
    if out is not None:
        q = out
    else:
        q = nf4_empty_single(rows, cols, W.device) if single_level else nf4_empty(rows, cols, W.device)
    st = q.c_struct()
    _abi.check(_abi.lib().qlora_nf4_quantize(_ptr(W), rows, cols, ctypes.byref(st),
                                             _stream(W.device)), "qlora_nf4_quantize")
    return q


def nf4_dequant(Wq: NF4Weight, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    if out is None:
        out = torch.empty(Wq.rows, Wq.cols, dtype=torch.bfloat16, device=Wq.codes.device)
    st = Wq.c_struct()
    _abi.check(_abi.lib().qlora_nf4_dequant(ctypes.byref(st), _ptr(out), _stream(out.device)),
               "qlora_nf4_dequant")
    return out


def workspace_bytes(M: int, N: int, K: int, r: int, dropout: bool = False) -> int:
    if dropout:
        return int(_abi.lib().qlora_linear_dropout_workspace_bytes(M, N, K, r))
    return int(_abi.lib().qlora_linear_workspace_bytes(M, N, K, r))


def make_workspace(M: int, N: int, K: int, r: int, device, dropout: bool = False) -> torch.Tensor:
    return torch.empty(workspace_bytes(M, N, K, r, dropout), dtype=torch.uint8, device=device)


def pack_keep_mask(keep: torch.Tensor) -> torch.Tensor:
    """A boolean [M, K] keep mask as the library's bit-packed form: element m K + k in
    bit (m K + k) mod 8 of byte (m K + k) / 8 (uint8 [M K / 8], on keep's device).
    Marshalling only (torch bit operations)."""
    if keep.dim() != 2 or keep.shape[1] % 8:
        raise ValueError("keep must be [M, K] with K a multiple of 8")
    bits = keep.reshape(-1, 8).to(torch.uint8)
    w = torch.tensor([1, 2, 4, 8, 16, 32, 64, 128], dtype=torch.uint8, device=keep.device)
    return (bits * w).sum(dim=1, dtype=torch.uint8).contiguous()


def _check_shapes(X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                  dY: Optional[torch.Tensor] = None) -> None:
    M, K = X.shape
    r = A.shape[1]
    if K != Wq.cols or A.shape[0] != Wq.cols or B.shape != (r, Wq.rows):
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, W [{Wq.rows}, {Wq.cols}], "
                         f"A {tuple(A.shape)}, B {tuple(B.shape)}")
    if dY is not None and dY.shape != (M, Wq.rows):
        raise ValueError(f"dY {tuple(dY.shape)} != ({M}, {Wq.rows})")


def linear_fwd(X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor, s: float,
               workspace: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
               XA: Optional[torch.Tensor] = None, want_xa: bool = True,
               keep_bits: Optional[torch.Tensor] = None, dropout_p: float = 0.0):
    """Y = X deq(W)^T + s (X A) B  (bf16 [M, N]);  returns (Y, XA fp32 [M, r] or None).
    With keep_bits (pack_keep_mask of the [M, K] keep mask) the adapter input is
    X (.) keep / (1 - dropout_p)."""
    X = _bf16_2d(X, "X")
    A = _bf16_2d(A, "A")
    B = _bf16_2d(B, "B")
    _check_shapes(X, Wq, A, B)
    M = X.shape[0]
    r = A.shape[1]
    dev = X.device
    if Y is None:
        Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=dev)
    if XA is None and want_xa:
        XA = torch.empty(M, r, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = make_workspace(M, Wq.rows, Wq.cols, r, dev, dropout=keep_bits is not None)
    st = Wq.c_struct()
    if keep_bits is None:
        _abi.check(_abi.lib().qlora_linear_fwd(
            _ptr(X), M, ctypes.byref(st), _ptr(A), _ptr(B), r, float(s), _ptr(Y), _ptr(XA),
            _ptr(workspace), workspace.numel(), _stream(dev)), "qlora_linear_fwd")
    else:
        _abi.check(_abi.lib().qlora_linear_fwd_ex(
            _ptr(X), M, ctypes.byref(st), _ptr(A), _ptr(B), r, float(s), _ptr(keep_bits), float(dropout_p),
            _ptr(Y), _ptr(XA), _ptr(workspace), workspace.numel(), _stream(dev)), "qlora_linear_fwd_ex")
    return Y, XA


def linear_bwd(dY: torch.Tensor, X: torch.Tensor, XA: Optional[torch.Tensor], Wq: NF4Weight,
               A: torch.Tensor, B: torch.Tensor, s: float, need_dx: bool = True,
               workspace: Optional[torch.Tensor] = None, dX: Optional[torch.Tensor] = None,
               dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
               keep_bits: Optional[torch.Tensor] = None, dropout_p: float = 0.0,
               accumulate: bool = False):
    """Returns (dX bf16 [M, K] or None, dA fp32 [K, r], dB fp32 [r, N]).  keep_bits /
    dropout_p as in linear_fwd; accumulate adds into the given dA and dB."""
    dY = _bf16_2d(dY, "dY")
    X = _bf16_2d(X, "X")
    A = _bf16_2d(A, "A")
    B = _bf16_2d(B, "B")
    _check_shapes(X, Wq, A, B, dY)
    M = X.shape[0]
    r = A.shape[1]
    dev = X.device
    if dX is None and need_dx:
        dX = torch.empty(M, Wq.cols, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(Wq.cols, r, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(r, Wq.rows, dtype=torch.float32, device=dev)
    if accumulate and (dA is None or dB is None):
        raise ValueError("accumulate needs the dA and dB to add into")
    if workspace is None:
        workspace = make_workspace(M, Wq.rows, Wq.cols, r, dev, dropout=keep_bits is not None)
    st = Wq.c_struct()
    if keep_bits is None and not accumulate:
        _abi.check(_abi.lib().qlora_linear_bwd(
            _ptr(dY), _ptr(X), _ptr(XA), M, ctypes.byref(st), _ptr(A), _ptr(B), r, float(s),
            _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(), _stream(dev)),
            "qlora_linear_bwd")
    else:
        _abi.check(_abi.lib().qlora_linear_bwd_ex(
            _ptr(dY), _ptr(X), _ptr(XA), M, ctypes.byref(st), _ptr(A), _ptr(B), r, float(s),
            _ptr(keep_bits), float(dropout_p), 1 if accumulate else 0,
            _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(), _stream(dev)),
            "qlora_linear_bwd_ex")
    return dX, dA, dB


def nf4_merge(A: torch.Tensor, B: torch.Tensor, s: float, Wq: Optional[NF4Weight] = None,
              W16: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The adapter folded into a 16-bit weight: bf16(base + s (A B)^T) [N, K], base the
    bf16 original W16 or the dequantized Wq (pass exactly one)."""
    A = _bf16_2d(A, "A")
    B = _bf16_2d(B, "B")
    if (Wq is None) == (W16 is None):
        raise ValueError("pass exactly one of Wq and W16")
    if W16 is not None:
        W16 = _bf16_2d(W16, "W16")
        N, K = W16.shape
        dev = W16.device
    else:
        N, K = Wq.rows, Wq.cols
        dev = Wq.codes.device
    r = A.shape[1]
    if A.shape[0] != K or tuple(B.shape) != (r, N):
        raise ValueError(f"shape mismatch: W [{N}, {K}], A {tuple(A.shape)}, B {tuple(B.shape)}")
    if out is None:
        out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    st = Wq.c_struct() if Wq is not None else None
    _abi.check(_abi.lib().qlora_nf4_merge(ctypes.byref(st) if st is not None else None, _ptr(W16), N, K,
                                          _ptr(A), _ptr(B), r, s, _ptr(out), _stream(dev)),
               "qlora_nf4_merge")
    return out


def device_status(sync_stream: bool = True) -> Tuple[int, int]:
    """(status code, flags) of the current device; reads and clears the word."""
    flags = ctypes.c_uint32(0)
    code = _abi.lib().qlora_get_device_status(_stream(), ctypes.byref(flags))
    return code, flags.value


def selftest_wait_timeout(timeout_us: int) -> int:
    return _abi.lib().qlora_selftest_wait_timeout(timeout_us, _stream())


def set_wait_limit_us(limit_us: int) -> int:
    return int(_abi.lib().qlora_set_wait_limit_us(limit_us))


def gemm_units() -> tuple:
    """(single CTAs, CTA pairs) the fused GEMM runs on this device."""
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    _abi.check(_abi.lib().qlora_gemm_units(ctypes.byref(a), ctypes.byref(b)), "qlora_gemm_units")
    return a.value, b.value


def set_gemm_pairing(enable: bool) -> bool:
    """Two-CTA (256-row) GEMM tiles where the output width allows; returns the previous setting."""
    return bool(_abi.lib().qlora_set_gemm_pairing(1 if enable else 0))


def profile_enable(on: bool = True) -> None:
    """Record CUDA events around every launch of the library's kernels."""
    _abi.check(_abi.lib().qlora_profile_enable(1 if on else 0), "qlora_profile_enable")


def profile_read():
    """[(kernel kind name, milliseconds)] of the launches recorded since enabling
    (oldest first, at most the ring capacity) and the total launch count."""
    cap = _abi.PROFILE_CAP
    kinds = (ctypes.c_int * cap)()
    ms = (ctypes.c_float * cap)()
    n = _abi.lib().qlora_profile_read(cap, kinds, ms)
    if n < 0:
        raise RuntimeError("qlora_profile_read failed")
    k = min(n, cap)
    return [(_abi.KERNEL_KINDS[kinds[i]], float(ms[i])) for i in range(k)], n
