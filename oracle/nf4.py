"""NF4 table, blockwise quantization with double quantization, dequantization.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Plain, slow, obviously
correct NumPy; no blocking or reordering beyond what the method states.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtri

BLOCK = 64          # values per first-level block ("QLoRA", ozercemkelahmet.com, How it works, Step 1)
GROUP = 256         # first-level constants per second-level constant (reading; see package docstring)
ZERO_CODE = 7       # index of the exact-zero level in the sorted table

# Upper quantile of the table construction: the mean of 1 - 1/32 and 1 - 1/30.
# A named constant (reading); the pages only place the levels at normal quantiles.
P_MAX = 0.5 * ((1.0 - 1.0 / 32.0) + (1.0 - 1.0 / 30.0))


# ---------------------------------------------------------------------------
# a1: the 16 NormalFloat levels
# ---------------------------------------------------------------------------
def nf4_levels_f64() -> np.ndarray:
    """16 levels at normal quantiles, each bin of (equal) probability mass, denser
    near zero, normalised to [-1, 1] with one exact zero.

    "QLoRA: Efficient Finetuning of Quantized LLMs" (crackai.dev), How It Works 1;
    "QLoRA" (ozercemkelahmet.com), How it works -- Why NormalFloat.

    Positive half: Phi^-1 at 9 evenly spaced probabilities in [0.5, P_MAX], the
    first (0.5 -> 0) dropped: 8 levels.  Negative half: -Phi^-1 at 8 evenly
    spaced probabilities in [0.5, P_MAX], first dropped: 7 levels.  Plus 0.
    Everything divided by max |level| = Phi^-1(P_MAX).
    """
    pos = ndtri(np.linspace(0.5, P_MAX, 9))[1:]
    neg = -ndtri(np.linspace(0.5, P_MAX, 8))[1:]
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    return v / np.max(np.abs(v))


def nf4_levels() -> np.ndarray:
    """The table as the fp32 constants the quantizer and dequantizer use."""
    return nf4_levels_f64().astype(np.float32)


# ---------------------------------------------------------------------------
# helpers: float32 / bf16 views
# ---------------------------------------------------------------------------
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_rn(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, nearest, ties to even (IEEE RN), as bits.

    Written as the plain definition: the two bf16 neighbours of x (truncation
    and the next one away from zero), pick the nearer, on a tie the one with an
    even last bit.  Differences are exact in fp64.
    """
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32)
    lo_bits = (u & np.uint32(0xFFFF0000))
    hi_bits = lo_bits + np.uint32(0x10000)
    lo = lo_bits.view(np.float32).astype(np.float64)
    hi = hi_bits.view(np.float32).astype(np.float64)
    xv = x.astype(np.float64)
    d_lo = np.abs(xv - lo)
    d_hi = np.abs(hi - xv)
    lo_even = ((lo_bits >> np.uint32(16)) & np.uint32(1)) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    out = np.where(take_hi, hi_bits, lo_bits) >> np.uint32(16)
    return out.astype(np.uint16)


def f64_to_bf16_rn(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 in ONE step, nearest, ties to even, as bits.

    Going through float32 first would round twice, which differs from one
    rounding when the fp32 step lands exactly on a bf16 tie.  Same plain
    definition as above, on the exact fp64 value: the bf16 quantum at x is
    2^(e-8) for x = m 2^e, m in [0.5, 1) (2^-133 below the normal range); the
    two neighbours are x truncated to a multiple of it and the next multiple
    away from zero; the nearer wins, a tie goes to the one with an even last
    bit.  Magnitudes that round to 2^128 or beyond give infinity.  Finite
    inputs only.
    """
    x = np.asarray(x, np.float64)
    shape = x.shape
    x = x.ravel()
    _, e = np.frexp(x)
    e = np.maximum(e, -125)                      # below 2^-126 the quantum stays 2^-133
    q = np.ldexp(1.0, e - 8)
    t = np.trunc(x / q)                          # exact: x / q only shifts the exponent
    lo = t * q
    hi = (t + np.sign(x)) * q
    d_lo = np.abs(x - lo)
    d_hi = np.abs(hi - x)
    lo_even = np.mod(np.abs(t), 2) == 0
    v = np.where((d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even), hi, lo)
    v = np.where(np.abs(v) >= 2.0 ** 128, np.copysign(np.inf, x), v)
    v = np.where(x == 0, x, v)                   # keeps the sign of a zero
    bits = (v.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return bits.reshape(shape)


# ---------------------------------------------------------------------------
# a2: block absmax
# ---------------------------------------------------------------------------
def block_absmax(w: np.ndarray) -> np.ndarray:
    """Largest absolute value of each 64-value block of the flattened tensor
    (row-major); the last block may be partial.

    "QLoRA" (ozercemkelahmet.com), How it works, Step 1 and "A worked example" 1.
    Exact (a max of float32 magnitudes): returned as float32.
    """
    w = np.asarray(w, np.float32).ravel()
    n = w.size
    nb = (n + BLOCK - 1) // BLOCK
    pad = np.zeros(nb * BLOCK, np.float32)
    pad[:n] = np.abs(w)
    return pad.reshape(nb, BLOCK).max(axis=1)


# ---------------------------------------------------------------------------
# a3: normalise, nearest level, pack
# ---------------------------------------------------------------------------
def nearest_level(xn: np.ndarray, levels: np.ndarray | None = None) -> np.ndarray:
    """Index of the nearest of the 16 levels to each float32 xn, ties to the lower
    index.  |xn - L_i| is formed in fp64, where it is exact for the candidates
    that can tie (both operands are float32 of nearby magnitude); argmin returns
    the first (lower) index on equality."""
    L = (nf4_levels() if levels is None else levels).astype(np.float64)
    x = np.asarray(xn, np.float32).astype(np.float64).ravel()
    out = np.empty(x.size, np.uint8)
    step = 1 << 20
    for i in range(0, x.size, step):
        d = np.abs(x[i:i + step, None] - L[None, :])
        out[i:i + step] = np.argmin(d, axis=1).astype(np.uint8)
    return out


def normalise(w: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """xn = RN32(w / a_b), IEEE float32 division; blocks with a_b = 0 give 0."""
    w = np.asarray(w, np.float32).ravel()
    a = np.repeat(absmax.astype(np.float32), BLOCK)[: w.size]
    safe = np.where(a > 0, a, np.float32(1.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        xn = (w / safe).astype(np.float32)
    return np.where(a > 0, xn, np.float32(0.0)).astype(np.float32)


def block_codes(w: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """4-bit code per element ("QLoRA", ozercemkelahmet.com, How it works, Step 1:
    each normalised value is mapped to the nearest of 16 levels)."""
    codes = nearest_level(normalise(w, absmax))
    a = np.repeat(absmax, BLOCK)[: codes.size]
    codes[a == 0] = ZERO_CODE
    return codes


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2j in bits 0-3, element 2j+1 in bits 4-7;
    an odd tail leaves the high nibble 0."""
    c = np.asarray(codes, np.uint8).ravel()
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, np.uint8)])
    return (c[0::2] | (c[1::2] << np.uint8(4))).astype(np.uint8)


def unpack_codes(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, np.uint8).ravel()
    out = np.empty(p.size * 2, np.uint8)
    out[0::2] = p & np.uint8(0x0F)
    out[1::2] = p >> np.uint8(4)
    return out[:n]


# ---------------------------------------------------------------------------
# a4: double quantization of the block constants
# ---------------------------------------------------------------------------
def double_quantize(absmax: np.ndarray):
    """8-bit codes for the per-block constants, in groups of 256, with one fp32
    second-level constant per group ("QLoRA", ozercemkelahmet.com, How it works,
    Step 3; crackai.dev, How It Works 2: constants go from 32 to 8 bits).

    Reading: a_b >= 0, so an unsigned linear code over [0, c_g] with
    step_g = RN32(c_g / 255) and q8_b = min(255, rint_even(RN32(a_b / step_g))).
    A group whose maximum is 0 stores step 0 and codes 0.
    """
    a = np.asarray(absmax, np.float32).ravel()
    nb = a.size
    ng = (nb + GROUP - 1) // GROUP
    step = np.zeros(ng, np.float32)
    q8 = np.zeros(nb, np.uint8)
    for g in range(ng):
        seg = a[g * GROUP:(g + 1) * GROUP]
        c = np.float32(seg.max())
        if c == 0:
            continue
        st = np.float32(c / np.float32(255.0))
        step[g] = st
        ratio = (seg / st).astype(np.float32)
        q = np.minimum(np.rint(ratio.astype(np.float64)), 255.0)
        q8[g * GROUP:(g + 1) * GROUP] = q.astype(np.uint8)
    return q8, step


def block_scales(q8: np.ndarray, step: np.ndarray) -> np.ndarray:
    """Reconstructed first-level constant per block: RN32(q8 * step_g)."""
    q8 = np.asarray(q8, np.uint8).ravel()
    g = np.arange(q8.size) // GROUP
    return (q8.astype(np.float32) * np.asarray(step, np.float32)[g]).astype(np.float32)


# ---------------------------------------------------------------------------
# full quantize / dequantize
# ---------------------------------------------------------------------------
def storage_bytes(n: int):
    """Bytes of (packed codes, 8-bit constants, fp32 second-level constants)."""
    nb = (n + BLOCK - 1) // BLOCK
    return (n + 1) // 2, nb, 4 * ((nb + GROUP - 1) // GROUP)


def quantize(w) -> dict:
    """Blockwise NF4 with double quantization of a float32 (or bf16-valued)
    tensor, flattened row-major.  Returns packed codes, q8, step and, for
    checking, the unquantized absmax and the unpacked codes."""
    w = np.asarray(w, np.float32).ravel()
    a = block_absmax(w)
    codes = block_codes(w, a)
    q8, step = double_quantize(a)
    return dict(n=w.size, codes=pack_codes(codes), q8=q8, step=step,
                absmax=a, codes_unpacked=codes)


def quantize_bf16(bits) -> dict:
    return quantize(bf16_to_f32(np.asarray(bits, np.uint16).ravel()))


def dequantize(packed, q8, step, n: int) -> np.ndarray:
    """bf16 bits of bf16_RN(RN32(L[code] * RN32(q8 * step))) per element
    ("QLoRA", ozercemkelahmet.com, "A worked example" 4: multiply levels by the
    block constant; Overview: into a compute type such as bfloat16)."""
    codes = unpack_codes(packed, n)
    L = nf4_levels()
    scale = np.repeat(block_scales(q8, step), BLOCK)[:n]
    prod = (L[codes] * scale).astype(np.float32)
    return f32_to_bf16_rn(prod)


# ---------------------------------------------------------------------------
# single-level variant: Steps 1-2 without Step 3
# ---------------------------------------------------------------------------
def storage_bytes_single_level(n: int):
    """Bytes of (packed codes, fp32 block constants) when the block constants are
    kept in fp32 ("QLoRA", ozercemkelahmet.com, How it works, Step 2: one 32-bit
    constant per 64 values, half a bit per weight)."""
    nb = (n + BLOCK - 1) // BLOCK
    return (n + 1) // 2, 4 * nb


def quantize_single_level(w) -> dict:
    """Blockwise NF4 with fp32 block constants (no double quantization): the
    codes of Steps 1-2, which use the unquantized absmax exactly as quantize()
    does, and the absmax itself as the stored constant."""
    w = np.asarray(w, np.float32).ravel()
    a = block_absmax(w)
    codes = block_codes(w, a)
    return dict(n=w.size, codes=pack_codes(codes), absmax=a, codes_unpacked=codes)


def dequantize_single_level(packed, absmax, n: int) -> np.ndarray:
    """bf16 bits of bf16_RN(RN32(L[code] * a_b)): the level times the block's
    stored fp32 constant, into the bf16 compute type."""
    codes = unpack_codes(packed, n)
    L = nf4_levels()
    scale = np.repeat(np.asarray(absmax, np.float32).ravel(), BLOCK)[:n]
    prod = (L[codes] * scale).astype(np.float32)
    return f32_to_bf16_rn(prod)
