"""GPU parity of NF4 quantize (+ double quant) and dequant against the oracle:
bit-exact codes, packed bytes, q8, step and dequantized bf16.  Calls go through
the C ABI (bit_nf4_quantized_19_b200 -> libqlora_nf4.so)."""
import numpy as np
import pytest

import helpers as H
from oracle import nf4 as onf4
from synth import (bf16_bits_from_f32, bf16_bits_to_f32, normal_bf16, heavy_tail_chunk,
                   CHUNK_ELEMS, n_chunks)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_19_b200 as q
    from bit_nf4_quantized_19_b200 import build
    build.build()
    return q


def _gpu_quant(q, bits, rows, cols):
    W = H.bits_to_dev(bits, (rows, cols))
    Wq = q.nf4_quantize(W)
    code, flags = q.device_status()
    return Wq, code, flags


def _check_quant(q, bits, rows, cols):
    Wq, code, flags = _gpu_quant(q, bits, rows, cols)
    assert code == 0 and flags == 0
    ref = H.oracle_quantize_bits(bits.ravel())
    got_codes = Wq.codes.cpu().numpy()
    assert np.array_equal(got_codes, ref["codes"]), "packed codes differ"
    assert np.array_equal(Wq.q8.cpu().numpy(), ref["q8"]), "q8 differs"
    assert np.array_equal(Wq.step.cpu().numpy().view(np.uint32), ref["step"].view(np.uint32)), "step differs"
    return Wq, ref


@pytest.mark.parametrize("rows,cols", [(1, 1), (1, 2), (1, 7), (1, 63), (1, 64), (1, 65), (3, 43),
                                       (1, 1000), (1, 16384), (1, 16385), (7, 7035), (128, 128),
                                       (1024, 1024)])
def test_quantize_bit_exact_sizes(q, rows, cols):
    bits = normal_bf16(0, f"qz{rows}x{cols}", (rows, cols), 0.02)
    _check_quant(q, bits, rows, cols)


def test_quantize_special_values(q):
    rng = np.random.default_rng(0)
    blocks = []
    blocks.append(np.zeros(64, np.float32))                                   # all-zero block
    z = np.zeros(64, np.float32); z[::3] = -0.0; blocks.append(z)            # negative zeros
    b = (rng.standard_normal(64) * 0.02).astype(np.float32); b[5] = 1.0; b[6] = -1.0
    blocks.append(b)                                                          # +-absmax
    blocks.append(np.full(64, 0.37, np.float32))                              # constant block
    blocks.append(np.full(64, -2.5, np.float32))
    blocks.append((rng.standard_normal(64) * 1e-39).astype(np.float32))      # subnormal bf16
    blocks.append((rng.standard_normal(64) * 3e38 / 8).astype(np.float32))    # huge
    L = onf4.nf4_levels()
    blocks.append((L[rng.integers(0, 16, 64)] * np.float32(0.5)).astype(np.float32))  # on grid
    w = np.concatenate(blocks + [(rng.standard_normal(64 * 300) * 0.02).astype(np.float32)])
    bits = bf16_bits_from_f32(w)
    _check_quant(q, bits, 1, bits.size)


def test_quantize_exhaustive_bf16_magnitudes(q):
    """Every finite bf16 value w with |w| <= a, for a sample of block maxima a:
    block = [a, 63 values], so every code decision of every bf16 input is covered."""
    rng = np.random.default_rng(1)
    all_bits = np.arange(0, 0x7F80, dtype=np.uint16)             # finite non-negative bf16
    mags = bf16_bits_to_f32(all_bits)
    a_bits = np.concatenate([rng.integers(0x0001, 0x7F7F, 24).astype(np.uint16),
                             np.array([0x3F80, 0x3C23, 0x0080, 0x0001, 0x7F7F], np.uint16)])
    rows = []
    for ab in a_bits:
        a = bf16_bits_to_f32(np.array([ab], np.uint16))[0]
        vals = all_bits[mags <= a]
        vals = np.concatenate([vals, vals | np.uint16(0x8000)])    # both signs
        pad = (-vals.size) % 63
        vals = np.concatenate([vals, np.zeros(pad, np.uint16)]).reshape(-1, 63)
        blk = np.concatenate([np.full((vals.shape[0], 1), ab, np.uint16), vals], axis=1)
        rows.append(blk.ravel())
    bits = np.concatenate(rows)
    _check_quant(q, bits, 1, bits.size)


@pytest.mark.parametrize("bad", [0x7F80, 0xFF80, 0x7FC0, 0xFFC1])   # +inf, -inf, quiet NaN, negative NaN
def test_nonfinite_input_sets_device_status(q, bad):
    bits = normal_bf16(0, "nonfinite", (1, 4096), 0.02)
    bits[0, 100] = bad
    Wq, code, flags = _gpu_quant(q, bits, 1, 4096)
    assert code == 6 and (flags & 2)
    code2, flags2 = q.device_status()
    assert code2 == 0 and flags2 == 0            # read-and-clear


def test_quantize_heavy_tail_64m(q):
    n = 4 * CHUNK_ELEMS
    bits = np.concatenate([heavy_tail_chunk(0, c, n) for c in range(4)])
    _check_quant(q, bits, 4096, n // 4096)


@pytest.mark.parametrize("n", [1, 15, 16, 17, 64 * 7 + 5, 16384 * 2 + 33, 1 << 20])
def test_dequant_bit_exact_random_codes(q, n):
    import torch
    rng = np.random.default_rng(n)
    cb, qb, sb = onf4.storage_bytes(n)
    codes = rng.integers(0, 256, cb, dtype=np.uint8)
    if n % 2:
        codes[-1] &= 0x0F
    q8 = rng.integers(0, 256, qb, dtype=np.uint8)
    step = (np.abs(rng.standard_normal(sb // 4)) * 1e-3).astype(np.float32)
    ref = onf4.dequantize(codes, q8, step, n)
    Wq = q.NF4Weight(torch.from_numpy(codes).cuda(), torch.from_numpy(q8).cuda(),
                     torch.from_numpy(step).cuda(), 1, n)
    out = q.nf4_dequant(Wq)
    assert np.array_equal(H.dev_to_bits(out).ravel(), ref)


def test_dequant_of_quantized_weight(q):
    bits = normal_bf16(3, "deqw", (512, 768), 0.02)
    ref = H.oracle_quantize_bits(bits.ravel())
    Wq, _, _ = _gpu_quant(q, bits, 512, 768)
    out = H.dev_to_bits(q.nf4_dequant(Wq)).ravel()
    assert np.array_equal(out, onf4.dequantize(ref["codes"], ref["q8"], ref["step"], bits.size))


def test_full_size_1e9_sampled(q):
    """The 1.0e9-element heavy-tailed tensor at full size (the bench's launch
    configuration); three chunks of 2^24 values regenerated on the host are
    checked bit-exactly for quantize and dequant."""
    import torch
    n = 1_000_000_000
    nc = n_chunks(n)
    W = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    for c in range(nc):
        ch = heavy_tail_chunk(0, c, n)
        W[c * CHUNK_ELEMS:c * CHUNK_ELEMS + ch.size].copy_(
            torch.from_numpy(ch.view(np.int16)).view(torch.bfloat16))
    Wq = q.nf4_quantize(W.view(1, n))
    out = q.nf4_dequant(Wq).view(-1)
    code, flags = q.device_status()
    assert code == 0
    for c in (0, nc // 2, nc - 1):
        lo = c * CHUNK_ELEMS
        ch = heavy_tail_chunk(0, c, n)
        ref = onf4.quantize_bf16(ch)
        g0, g1 = lo // 16384, (lo + ch.size + 16383) // 16384
        assert np.array_equal(Wq.codes[lo // 2:(lo + ch.size + 1) // 2].cpu().numpy(), ref["codes"])
        assert np.array_equal(Wq.q8[lo // 64:(lo + ch.size + 63) // 64].cpu().numpy(), ref["q8"])
        assert np.array_equal(Wq.step[g0:g1].cpu().numpy().view(np.uint32), ref["step"].view(np.uint32))
        deq_ref = onf4.dequantize(ref["codes"], ref["q8"], ref["step"], ch.size)
        assert np.array_equal(H.dev_to_bits(out[lo:lo + ch.size]), deq_ref)
    del W, Wq, out
    torch.cuda.empty_cache()
