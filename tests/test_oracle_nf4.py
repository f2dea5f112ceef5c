"""Pins for the NF4 oracle: what the pages and the mathematics fix, checked by
routes independent of the oracle's own arithmetic (exact rationals, stdlib erf,
closed forms, printed figures, torch's bf16 conversion)."""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4
from synth import bf16_bits_from_f32, bf16_bits_to_f32


# ---------------------------------------------------------------- helpers
def phi(z):
    """Standard normal CDF from the stdlib (independent of scipy)."""
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def phi_inv_bisect(p):
    """Inverse normal CDF by bisection on math.erfc, to full double precision."""
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if phi(mid) < p:
            lo = mid
        else:
            hi = mid
        if hi - lo <= 0:
            break
    return 0.5 * (lo + hi)


def rn32_fraction(q: Fraction) -> np.float32:
    """Exact round-to-nearest-even of a rational to float32 (normals and
    subnormals), by integer arithmetic only."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    m = a / ulp
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * float(fl * ulp))


def brute_code(w: np.float32, a: np.float32, levels) -> int:
    """Code by brute force over all 16 levels in exact rational arithmetic."""
    if a == 0:
        return 7
    xn = Fraction(float(rn32_fraction(Fraction(float(w)) / Fraction(float(a)))))
    best, best_d = None, None
    for i, L in enumerate(levels):
        d = abs(xn - Fraction(float(L)))
        if best_d is None or d < best_d:  # strict: ties keep the lower index
            best, best_d = i, d
    return best


# ---------------------------------------------------------------- a1 table
def test_table_shape_monotone_exact_ends():
    L = nf4.nf4_levels()
    assert L.dtype == np.float32 and L.size == 16
    assert np.all(np.diff(L.astype(np.float64)) > 0)
    assert L[0] == -1.0 and L[15] == 1.0 and L[7] == 0.0
    assert (L < 0).sum() == 7 and (L > 0).sum() == 8      # asymmetric halves


def test_table_denser_near_zero():
    L = nf4.nf4_levels().astype(np.float64)
    gaps = np.diff(L)
    # spacing grows away from zero on both sides (denser levels near zero)
    assert np.all(np.diff(gaps[7:]) > 0) and np.all(np.diff(gaps[:7]) < 0)


def test_table_matches_independent_inverse_cdf_bitwise():
    """Rebuild the table with a bisection inverse CDF on math.erfc."""
    zmax = phi_inv_bisect(nf4.P_MAX)
    pos = [phi_inv_bisect(0.5 + k * (nf4.P_MAX - 0.5) / 8) for k in range(1, 9)]
    neg = [-phi_inv_bisect(0.5 + k * (nf4.P_MAX - 0.5) / 7) for k in range(1, 8)]
    ref = np.array(sorted(neg + [0.0] + pos)) / zmax
    assert np.array_equal(ref.astype(np.float32), nf4.nf4_levels())


def test_table_is_evenly_spaced_in_probability():
    """Each half sits at evenly spaced normal quantiles (checked with Phi)."""
    zmax = phi_inv_bisect(nf4.P_MAX)
    L64 = nf4.nf4_levels_f64()
    for k, i in enumerate(range(8, 16), start=1):
        assert abs(phi(L64[i] * zmax) - (0.5 + k * (nf4.P_MAX - 0.5) / 8)) < 1e-12
    for k, i in enumerate(range(6, -1, -1), start=1):
        assert abs(phi(-L64[i] * zmax) - (0.5 + k * (nf4.P_MAX - 0.5) / 7)) < 1e-12


def test_equal_mass_per_bin_analytic():
    """For N(0,1) scaled by 1/Phi^-1(P_MAX), every nearest-level bin holds about
    1/16 of the probability (within +-20%)."""
    zmax = phi_inv_bisect(nf4.P_MAX)
    L = nf4.nf4_levels().astype(np.float64)
    edges = np.concatenate([[-np.inf], 0.5 * (L[1:] + L[:-1]), [np.inf]])
    mass = [phi(edges[i + 1] * zmax) - phi(edges[i] * zmax) for i in range(16)]
    assert abs(sum(mass) - 1.0) < 1e-12
    for m in mass:
        assert 0.8 / 16 <= m <= 1.2 / 16, mass


def test_equal_mass_per_bin_sampled():
    rng = np.random.default_rng(1234)
    z = rng.standard_normal(1_000_000)
    zmax = phi_inv_bisect(nf4.P_MAX)
    x = np.clip(z / zmax, -1, 1).astype(np.float32)
    codes = nf4.nearest_level(x)
    frac = np.bincount(codes, minlength=16) / codes.size
    assert np.all(frac > 0.8 / 16) and np.all(frac < 1.2 / 16), frac


# ---------------------------------------------------------------- worked example
def test_worked_example(golden):
    g = golden("worked_example.txt")
    blk = np.array(g["block"], np.float32)
    q = nf4.quantize(blk)
    # step 1: absmax and the normalised block (exact arithmetic; float32 inputs)
    assert abs(float(q["absmax"][0]) - g["absmax"]) < 1e-7
    xn = nf4.normalise(blk, q["absmax"])
    np.testing.assert_allclose(xn, g["normalised"], rtol=0, atol=1e-7)
    L = nf4.nf4_levels()
    lv = L[q["codes_unpacked"]]
    # step 2 is a hypothetical on the page: three of the four agree with the
    # NF4 levels to 0.02; for 0.125 the nearest NF4 level is 0.1609, not 0.1.
    sup = np.array(g["supposed"])
    assert np.all(np.abs(lv[1:] - sup[1:]) < 0.02)
    assert abs(lv[0] - 0.16093) < 1e-4 and abs(0.125 - lv[0]) < abs(0.125 - L[q["codes_unpacked"][0] - 1])
    # step 4: level * constant, "about" the printed values (same three elements)
    deq = nf4.bf16_to_f32(nf4.dequantize(q["codes"], q["q8"], q["step"], 4))
    assert np.all(np.abs(deq[1:] - np.array(g["about"][1:])) < 0.01)
    # the block stores four 4-bit indices (two bytes) plus the constant
    assert q["codes"].size == 2 and q["q8"].size == 1


# ---------------------------------------------------------------- a3 codes: brute force
def _random_blocks(rng, nblocks):
    L = nf4.nf4_levels()
    out = []
    for b in range(nblocks):
        kind = b % 6
        if kind == 0:
            w = rng.standard_normal(64).astype(np.float32) * np.float32(0.02)
        elif kind == 1:   # bf16-valued
            w = bf16_bits_to_f32(bf16_bits_from_f32(rng.standard_normal(64).astype(np.float32)))
        elif kind == 2:   # on-grid: exactly the levels times a power of two
            w = (L[rng.integers(0, 16, 64)] * np.float32(2.0 ** rng.integers(-20, 5))).astype(np.float32)
        elif kind == 3:   # exact midpoints between levels where float32 holds them
            mids = (L[1:].astype(np.float64) + L[:-1]) / 2
            m32 = mids.astype(np.float32)
            rep = m32[m32.astype(np.float64) == mids]
            w = rep[rng.integers(0, rep.size, 64)].astype(np.float32)
            w[0] = 1.0
        elif kind == 4:   # tiny / subnormal magnitudes, signed zeros
            w = (rng.standard_normal(64) * 1e-39).astype(np.float32)
            w[:4] = [0.0, -0.0, 1e-45, -1e-45]
        else:             # zero block
            w = np.zeros(64, np.float32)
            w[3] = -0.0
        out.append(w)
    return out


def test_codes_brute_force_exact_rationals():
    rng = np.random.default_rng(7)
    L = nf4.nf4_levels()
    blocks = _random_blocks(rng, 60)
    w = np.concatenate(blocks)
    q = nf4.quantize(w)
    codes = q["codes_unpacked"]
    for b, blk in enumerate(blocks):
        a = np.float32(np.max(np.abs(blk)))
        assert q["absmax"][b] == a
        for i in range(64):
            assert codes[b * 64 + i] == brute_code(blk[i], a, L), (b, i, blk[i], a)


def test_ties_go_to_lower_index():
    L = nf4.nf4_levels().astype(np.float64)
    mids = (L[1:] + L[:-1]) / 2
    exact = [i for i, m in enumerate(mids) if float(np.float32(m)) == m]
    assert exact, "some midpoints must be float32-representable for this pin"
    for i in exact:
        blk = np.zeros(64, np.float32)
        blk[0] = 1.0
        blk[1] = np.float32(mids[i])
        assert nf4.quantize(blk)["codes_unpacked"][1] == i


def test_special_values():
    blk = np.array([0.5, -0.5, -0.0, 0.0, 0.25, 1e-30] + [0.1] * 58, np.float32)
    c = nf4.quantize(blk)["codes_unpacked"]
    assert c[0] == 15 and c[1] == 0 and c[2] == 7 and c[3] == 7 and c[5] == 7
    z = nf4.quantize(np.zeros(64, np.float32))
    assert np.all(z["codes_unpacked"] == 7) and z["q8"][0] == 0 and z["step"][0] == 0


def test_on_grid_round_trip_codes():
    """Values already on the grid (levels times a power of two, in bf16) map
    back to their own level index."""
    rng = np.random.default_rng(3)
    L = nf4.nf4_levels()
    for k in (-12, -6, -1, 0, 3):
        idx = rng.integers(0, 16, 64)
        idx[0] = 15
        vals = bf16_bits_to_f32(bf16_bits_from_f32((L[idx] * np.float32(2.0 ** k)).astype(np.float32)))
        q = nf4.quantize(vals)
        assert np.array_equal(q["codes_unpacked"], idx.astype(np.uint8))


def test_packing_nibble_order_and_odd_tail():
    codes = np.array([1, 2, 3, 4, 15], np.uint8)
    p = nf4.pack_codes(codes)
    assert p.tolist() == [0x21, 0x43, 0x0F]
    assert nf4.unpack_codes(p, 5).tolist() == codes.tolist()


# ---------------------------------------------------------------- a4 double quant
def test_double_quant_closed_form_bits(golden):
    g = golden("memory_figures.txt")
    single = g["first_level_bits"] / g["block_values"]
    assert single == g["single_overhead_bits"] == 0.5
    for groups in (1, 3, 64):
        n = nf4.BLOCK * nf4.GROUP * groups
        cb, qb, sb = nf4.storage_bytes(n)
        bits = 8.0 * (cb + qb + sb) / n
        assert bits == 4.126953125
        overhead = bits - 4.0
        assert overhead == g["second_level_bits"] / 64 + 32 / (64 * 256)
        assert abs((single - overhead) - g["double_saving_bits"]) < 0.005
        # the actual quantize output has exactly these sizes
        if groups == 1:
            q = nf4.quantize(np.random.default_rng(0).standard_normal(n).astype(np.float32))
            assert (q["codes"].nbytes, q["q8"].nbytes, q["step"].nbytes) == (cb, qb, sb)


def test_storage_partial_last_group_1e9():
    cb, qb, sb = nf4.storage_bytes(1_000_000_000)
    assert cb == 500_000_000 and qb == 15_625_000 and sb == 4 * 61036
    assert 15_625_000 - 61035 * 256 == 40      # the last group holds 40 constants


def test_memory_figures_on_the_pages(golden):
    g = golden("memory_figures.txt")
    for p, g16, g4 in ((g["params_7b"], g["gb_7b_16bit"], g["gb_7b_4bit"]),
                       (g["params_65b"], g["gb_65b_16bit"], g["gb_65b_4bit"])):
        assert abs(2 * p / 1e9 - g16) / g16 < 0.01
        cb, qb, sb = nf4.storage_bytes(int(p))
        gb = (cb + qb + sb) / 1e9
        assert g4 <= gb <= g4 * 1.05        # "plus small overhead"


def test_double_quant_error_bound_and_max_code():
    rng = np.random.default_rng(11)
    a = np.abs(rng.standard_normal(256 * 5 + 17)).astype(np.float32) * np.float32(0.05)
    a[256 * 2:256 * 3] = 0.0                      # an all-zero group
    q8, step = nf4.double_quantize(a)
    sc = nf4.block_scales(q8, step)
    for g in range(step.size):
        seg = slice(g * 256, (g + 1) * 256)
        if a[seg].max() == 0:
            assert step[g] == 0 and np.all(q8[seg] == 0)
            continue
        assert q8[seg][np.argmax(a[seg])] == 255
        err = np.abs(sc[seg].astype(np.float64) - a[seg])
        assert np.all(err <= 0.5 * step[g] * (1 + 1e-6) + 4 * np.spacing(a[seg]))
        # monotone code
        o = np.argsort(a[seg], kind="stable")
        assert np.all(np.diff(q8[seg][o].astype(int)) >= 0)


def test_double_quant_values_exact_rationals():
    """q8 = min(255, round_half_even(RN32(a / RN32(c / 255)))) by exact rationals."""
    rng = np.random.default_rng(5)
    a = np.abs(rng.standard_normal(300)).astype(np.float32) * np.float32(0.03)
    q8, step = nf4.double_quantize(a)
    for g in range(step.size):
        seg = a[g * 256:(g + 1) * 256]
        c = Fraction(float(seg.max()))
        st = rn32_fraction(c / 255)
        assert st == step[g]
        for i, v in enumerate(seg):
            r = Fraction(float(rn32_fraction(Fraction(float(v)) / Fraction(float(st)))))
            fl = r.numerator // r.denominator
            rem = r - fl
            qq = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2) else 0)
            assert q8[g * 256 + i] == min(255, qq)


# ---------------------------------------------------------------- a5 dequant
def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(200_000) * 10.0 ** rng.integers(-30, 30, 200_000)).astype(np.float32)
    # exact ties: bf16 values with the 16th bit set
    ties = (bf16_bits_to_f32(bf16_bits_from_f32(x[:1000])).view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 1e-45, -3e-39], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nf4.f32_to_bf16_rn(x), ref)


def test_dequant_definition_by_hand():
    L = nf4.nf4_levels()
    packed = np.array([0x2F], np.uint8)         # codes 15, 2
    q8 = np.array([200], np.uint8)
    step = np.array([0.001], np.float32)
    out = nf4.bf16_to_f32(nf4.dequantize(packed, q8, step, 2))
    scale = np.float32(np.float32(200.0) * np.float32(0.001))
    for j, c in enumerate((15, 2)):
        prod = np.float32(L[c] * scale)
        import torch
        ref = torch.tensor([float(prod)], dtype=torch.float32).to(torch.bfloat16).float().item()
        assert out[j] == np.float32(ref)


def test_dequant_round_trip_error_bound():
    """|deq(w) - w| <= half the local level gap times the block constant, plus
    the double-quant and bf16 rounding."""
    rng = np.random.default_rng(2)
    w = bf16_bits_to_f32(bf16_bits_from_f32((rng.standard_normal(64 * 300) * 0.02).astype(np.float32)))
    q = nf4.quantize(w)
    d = nf4.bf16_to_f32(nf4.dequantize(q["codes"], q["q8"], q["step"], w.size)).astype(np.float64)
    L = nf4.nf4_levels().astype(np.float64)
    maxgap = np.max(np.diff(L))
    a = np.repeat(q["absmax"], 64).astype(np.float64)
    st = np.repeat(q["step"][np.arange(q["q8"].size) // 256], 64)
    bound = 0.5 * maxgap * a + 0.5 * st + np.abs(d) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(d - w) <= bound)
