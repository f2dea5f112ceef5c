"""Seeded input generators (numpy Philox-backed ``default_rng``).

Every tensor is produced as bf16 *bit patterns* (``uint16``) so that the device
copy and the oracle copy are the same bytes.  Draws are chunked with per-chunk
seeds ``(seed, tag, chunk)`` so that any chunk of a very large tensor can be
regenerated on its own (used for sampled parity checks at full size).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

# 2**24 elements per independently seeded chunk: a whole number of 16384-element
# groups, so a chunk never splits a quantization group.
CHUNK_ELEMS = 1 << 24


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (round to nearest, ties to even);
    returns the uint16 bit patterns.  Used only to store generated inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _tag_id(tag: str) -> int:
    # stable small integer from a tag string (no hashing randomness)
    return sum((i + 1) * ord(c) for i, c in enumerate(tag)) & 0xFFFFFF


def normal_bf16(seed: int, tag: str, shape, std: float) -> np.ndarray:
    """bf16 bits of std * N(0, 1), drawn in float32 then rounded to bf16."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    tid = _tag_id(tag)
    for c in range(0, max(1, (n + CHUNK_ELEMS - 1) // CHUNK_ELEMS)):
        lo = c * CHUNK_ELEMS
        hi = min(n, lo + CHUNK_ELEMS)
        if hi <= lo:
            break
        g = np.random.default_rng([seed, tid, c])
        z = g.standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = bf16_bits_from_f32(z * np.float32(std))
    return out.reshape(shape)


def normal_bf16_rows(seed: int, tag: str, shape, std: float, rows: int) -> np.ndarray:
    """The first `rows` rows of ``normal_bf16(seed, tag, shape, std)`` (a 2-D shape),
    bit for bit, drawing only the chunks that hold them."""
    R, C = shape
    rows = min(rows, R)
    n = rows * C
    out = np.empty(n, dtype=np.uint16)
    tid = _tag_id(tag)
    for c in range(0, (n + CHUNK_ELEMS - 1) // CHUNK_ELEMS):
        lo = c * CHUNK_ELEMS
        hi_full = min(R * C, lo + CHUNK_ELEMS)
        g = np.random.default_rng([seed, tid, c])
        z = g.standard_normal(hi_full - lo, dtype=np.float32)
        hi = min(n, hi_full)
        out[lo:hi] = bf16_bits_from_f32(z[: hi - lo] * np.float32(std))
    return out.reshape(rows, C)


def linear_problem_rows(M: int, N: int, K: int, r: int, alpha: float, w_std: float,
                        tokens: int, wrows: int, seed: int = 0) -> LinearProblem:
    """The leading part of ``linear_problem(M, N, K, r, alpha, w_std, seed)``: the
    first `wrows` rows of W, the first `tokens` rows of X and dY, and A and B whole,
    each bit-identical to the full problem's."""
    tag = f"{M}x{N}x{K}r{r}"
    W = normal_bf16_rows(seed, "W" + tag, (N, K), w_std, wrows)
    X = normal_bf16_rows(seed, "X" + tag, (M, K), 1.0, tokens)
    A = normal_bf16(seed, "A" + tag, (K, r), 1.0 / r)
    B = normal_bf16(seed, "B" + tag, (r, N), 0.01)
    dY = normal_bf16_rows(seed, "dY" + tag, (M, N), 1.0, tokens)
    return LinearProblem(tag + f"[:{tokens}]", tokens, N, K, r, alpha, W, X, A, B, dY)


def keep_mask(seed: int, tag: str, shape, p: float) -> np.ndarray:
    """A dropout keep mask: True with probability 1 - p per element, independently
    (drawn as uniform fp32 < 1 - p)."""
    g = np.random.default_rng([seed, _tag_id("keep" + tag), 0])
    return g.random(shape, dtype=np.float32) < np.float32(1.0 - p)


def n_chunks(n: int) -> int:
    return (n + CHUNK_ELEMS - 1) // CHUNK_ELEMS


def heavy_tail_chunk(seed: int, chunk: int, n_total: int, std: float = 0.02,
                     p_outlier: float = 1e-3, factor: float = 8.0) -> np.ndarray:
    """One chunk (``CHUNK_ELEMS`` elements, shorter at the end) of the large
    heavy-tailed tensor: std * N(0,1), each element independently multiplied by
    ``factor`` with probability ``p_outlier``.  Returns bf16 bits."""
    lo = chunk * CHUNK_ELEMS
    hi = min(n_total, lo + CHUNK_ELEMS)
    g = np.random.default_rng([seed, _tag_id("heavy"), chunk])
    z = g.standard_normal(hi - lo, dtype=np.float32) * np.float32(std)
    mask = g.random(hi - lo, dtype=np.float32) < np.float32(p_outlier)
    z[mask] *= np.float32(factor)
    return bf16_bits_from_f32(z)


@dataclasses.dataclass
class LinearProblem:
    """One adapted linear layer: W [N, K], X [M, K], A [K, r], B [r, N], dY [M, N]
    (all bf16 bits), rank r and LoRA scale s = alpha / r."""
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    W: np.ndarray
    X: np.ndarray
    A: np.ndarray
    B: np.ndarray
    dY: np.ndarray

    @property
    def s(self) -> float:
        return float(self.alpha) / float(self.r)


# name -> (W std, A std rule, list of (M, N, K)), r, alpha
WORKLOADS: Dict[str, dict] = {
    "small": dict(w_std=0.02, r=8, alpha=16.0, shapes=[(16, 1024, 1024)]),
    "llama7b": dict(w_std=0.02, r=16, alpha=32.0,
                    shapes=[(4096, 4096, 4096), (4096, 11008, 4096), (4096, 4096, 11008)]),
    "skinny": dict(w_std=0.02, r=16, alpha=32.0,
                   shapes=[(m, n, 4096) for n in (4096, 11008) for m in (1, 4, 16)]),
    "llama65b": dict(w_std=0.015, r=64, alpha=16.0,
                     shapes=[(8192, 8192, 8192), (8192, 22016, 8192), (8192, 8192, 22016)]),
}


def linear_problem(M: int, N: int, K: int, r: int, alpha: float, w_std: float,
                   seed: int = 0, name: str = "", with_dy: bool = True) -> LinearProblem:
    """Seeded inputs for one adapted linear layer.  A ~ N(0, 1/r) (std), B ~
    N(0, 0.01), X and dY ~ N(0, 1), W ~ N(0, w_std)."""
    tag = f"{M}x{N}x{K}r{r}"
    W = normal_bf16(seed, "W" + tag, (N, K), w_std)
    X = normal_bf16(seed, "X" + tag, (M, K), 1.0)
    A = normal_bf16(seed, "A" + tag, (K, r), 1.0 / r)
    B = normal_bf16(seed, "B" + tag, (r, N), 0.01)
    dY = normal_bf16(seed, "dY" + tag, (M, N), 1.0) if with_dy else np.zeros((0, N), np.uint16)
    return LinearProblem(name or tag, M, N, K, r, alpha, W, X, A, B, dY)


def workload_problems(name: str, seed: int = 0) -> List[LinearProblem]:
    w = WORKLOADS[name]
    return [linear_problem(M, N, K, w["r"], w["alpha"], w["w_std"], seed=seed,
                           name=f"{name}:{M}x{N}x{K}") for (M, N, K) in w["shapes"]]


def shapes_of(name: str) -> List[Tuple[int, int, int]]:
    return list(WORKLOADS[name]["shapes"])
