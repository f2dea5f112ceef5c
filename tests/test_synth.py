"""The seeded input generators shared by the tests, the oracle checks and the bench:
reproducible, chunk-stable (a chunk of a large tensor does not depend on the
tensor's length, so full-size sampled checks can regenerate it alone), rounded
to bf16 the same way as the oracle's independent rounding, and drawn with the
stated distributions."""
import numpy as np

from oracle import nf4 as onf4
from synth import CHUNK_ELEMS, bf16_bits_from_f32, heavy_tail_chunk, linear_problem, normal_bf16


def test_reproducible_and_seed_dependent():
    a = linear_problem(17, 384, 256, 8, 16.0, 0.02, seed=3)
    b = linear_problem(17, 384, 256, 8, 16.0, 0.02, seed=3)
    c = linear_problem(17, 384, 256, 8, 16.0, 0.02, seed=4)
    for name in ("W", "X", "A", "B", "dY"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
        assert not np.array_equal(getattr(a, name), getattr(c, name)), name
    assert not np.array_equal(a.X, a.dY)         # different tags draw different numbers


def test_chunks_do_not_depend_on_the_tensor_length():
    head = normal_bf16(1, "Wchunk", (CHUNK_ELEMS,), 0.02)
    longer = normal_bf16(1, "Wchunk", (CHUNK_ELEMS + 1000,), 0.02)
    assert np.array_equal(longer[:CHUNK_ELEMS], head)
    n_total = 3 * CHUNK_ELEMS + 5
    last = heavy_tail_chunk(2, 3, n_total)
    assert last.size == 5
    assert np.array_equal(heavy_tail_chunk(2, 1, n_total), heavy_tail_chunk(2, 1, 2 * CHUNK_ELEMS))


def test_bf16_rounding_matches_the_oracle():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(1 << 20) * np.exp(rng.uniform(-30, 30, 1 << 20))).astype(np.float32)
    assert np.array_equal(bf16_bits_from_f32(x), onf4.f32_to_bf16_rn(x))


def test_distributions():
    w = onf4.bf16_to_f32(normal_bf16(5, "dist", (1 << 20,), 0.02)).astype(np.float64)
    assert abs(w.mean()) < 1e-4 and abs(w.std() / 0.02 - 1) < 0.01
    h = onf4.bf16_to_f32(heavy_tail_chunk(5, 0, 1 << 22)).astype(np.float64)
    # beyond 6 sigma: N(0,1) alone gives ~2e-9; an outlier (p = 1e-3, x8) lands there when
    # |z| > 0.75, i.e. 45% of the time, so ~4.5e-4 of the values (+-1e-5 at this size)
    frac = np.mean(np.abs(h) > 6 * 0.02)
    assert 3.5e-4 < frac < 5.5e-4


def test_row_prefix_generators_match_the_full_tensors():
    """normal_bf16_rows / linear_problem_rows give the leading rows of the full
    tensors bit for bit, also when the rows span more than one seeded chunk."""
    from synth import CHUNK_ELEMS, linear_problem, linear_problem_rows, normal_bf16, normal_bf16_rows
    full = normal_bf16(3, "prefix", (3000, 8192), 0.5)
    rows = CHUNK_ELEMS // 8192 + 52                  # crosses the first chunk boundary
    assert np.array_equal(normal_bf16_rows(3, "prefix", (3000, 8192), 0.5, rows), full[:rows])
    assert np.array_equal(normal_bf16_rows(3, "prefix", (3000, 8192), 0.5, 5000), full)
    p = linear_problem(40, 96, 128, 8, 16.0, 0.02, seed=2)
    s = linear_problem_rows(40, 96, 128, 8, 16.0, 0.02, 7, 33, seed=2)
    assert np.array_equal(s.W, p.W[:33]) and np.array_equal(s.X, p.X[:7])
    assert np.array_equal(s.dY, p.dY[:7]) and np.array_equal(s.A, p.A) and np.array_equal(s.B, p.B)


def test_keep_mask_rate_and_packing():
    """keep_mask keeps each element with probability 1 - p; the binding's packer
    (bit-packed, element i in bit i mod 8 of byte i / 8) agrees with numpy's."""
    import torch
    from synth import keep_mask
    from bit_nf4_quantized_19_b200.api import pack_keep_mask
    k = keep_mask(0, "rate", (1000, 1024), 0.1)
    assert abs(k.mean() - 0.9) < 0.002
    assert not np.array_equal(k, keep_mask(1, "rate", (1000, 1024), 0.1))
    assert np.array_equal(k, keep_mask(0, "rate", (1000, 1024), 0.1))
    got = pack_keep_mask(torch.from_numpy(k[:37, :64])).numpy()
    assert np.array_equal(got, np.packbits(k[:37, :64].astype(np.uint8).ravel(), bitorder="little"))
    e = np.zeros((1, 8), bool)
    e[0, 3] = True
    assert pack_keep_mask(torch.from_numpy(e)).tolist() == [8]
