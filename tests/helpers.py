"""Shared helpers for the GPU parity tests (host <-> device bf16 bits, oracle
reference computations).  Inputs always come from ``synth``; expected values
always come from ``oracle``."""
from __future__ import annotations

import numpy as np

from oracle import linear as olin
from oracle import nf4 as onf4


def torch_mod():
    import torch
    return torch


def bits_to_dev(bits: np.ndarray, shape=None):
    torch = torch_mod()
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    t = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
    if shape is not None:
        t = t.reshape(shape)
    return t.cuda()


def dev_to_bits(t) -> np.ndarray:
    torch = torch_mod()
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_quantize_bits(bits: np.ndarray) -> dict:
    return onf4.quantize_bf16(bits)


def oracle_deq_bits(bits: np.ndarray) -> np.ndarray:
    q = onf4.quantize_bf16(bits)
    return onf4.dequantize(q["codes"], q["q8"], q["step"], bits.size).reshape(bits.shape)


def bf16_ulp_check(got_bits: np.ndarray, ref: np.ndarray, contraction: int) -> float:
    """Largest |got - ref| / (ulp_bf16(ref) + floor); <= 1 means every element is
    within one bf16 ulp of the exact value.  The absolute floor covers results
    that cancel to near zero, where fp32 accumulation noise dominates: about
    sqrt(K) * 2^-23 * rms(ref) for a K-term sum (truncating tensor-core
    accumulation), taken at 4 sigma."""
    rms_floor = 4.0 * np.sqrt(float(contraction)) * 2.0 ** -23
    got = onf4.bf16_to_f32(got_bits).astype(np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.abs(ref)
    e = np.floor(np.log2(np.maximum(mag, 1e-38)))
    ulp = 2.0 ** (e - 7)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return float(np.max(np.abs(got - ref) / (ulp + rms_floor * rms)))


# Element-wise bound of the fp32 rank-r outputs (XA, G, dA, dB), relative to the
# matching product of magnitudes (for dA: s |X|^T |G|).  The operands of those
# products are exact bf16 values or fp32 values carried as bf16 hi + lo pairs, which
# represent them to 2^-17 relative; fp32 accumulation adds far less than that on
# sums of random sign.  2^-15 leaves a factor 4.  A wrong row, column or split sum
# shows up at order 1 / sqrt(contraction) of the magnitude, far above it.
MAG_TOL = 2.0 ** -15


def mag_check(got, ref, mag) -> float:
    """Largest |got - ref| / (MAG_TOL * mag); <= 1 passes.  `mag` is the fp64
    product of the operands' magnitudes for each output element."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.asarray(mag, np.float64)
    floor = 1e-30
    return float(np.max(np.abs(got - ref) / (MAG_TOL * mag + floor)))


def lora_magnitudes(X, A, B, dY, s, XA=None, G=None):
    """Magnitude products for XA, G, dA and dB (fp64; inputs bf16 bits, or fp64 for
    XA and G when given)."""
    Xa, Aa, Ba, dYa = (np.abs(olin.as_f64(t)) for t in (X, A, B, dY))
    XAm = np.abs(np.asarray(XA, np.float64)) if XA is not None else Xa @ Aa
    Gm = np.abs(np.asarray(G, np.float64)) if G is not None else dYa @ Ba.T
    return dict(XA=Xa @ Aa, G=dYa @ Ba.T, dA=abs(s) * (Xa.T @ Gm), dB=abs(s) * (XAm.T @ dYa))


rel_fro = olin.rel_fro
