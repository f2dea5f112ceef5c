"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module only draws random numbers and stores them as bf16 bit patterns.  It
holds none of the quantization or linear-layer arithmetic: the oracle
(``oracle/``) and the CUDA library each implement the method on their own; both
receive the very same input bytes from here.

Workloads (all seeded, all synthetic; shapes and distributions of the QLoRA
linear-layer workloads, W stored ``[N, K]`` = out x in):

* ``small``:   W 1024x1024 ~N(0, 0.02), X 16x1024 ~N(0,1), r=8, alpha=16,
               A ~N(0, 1/8), B ~N(0, 0.01), dY ~N(0, 1).
* ``llama7b``: W 4096x4096, 11008x4096, 4096x11008 ~N(0, 0.02), 4096 tokens,
               r=16, alpha=32, A ~N(0, 1/16), B ~N(0, 0.01).
* ``skinny``:  W 4096x4096, 11008x4096, M in {1, 4, 16} tokens, r=16, fwd only.
* ``llama65b``: W 8192x8192, 22016x8192, 8192x22016 ~N(0, 0.015), 8192 tokens, r=64,
               alpha=16, A ~N(0, 1/64), B ~N(0, 0.01).
* ``tensor1e9``: 1.0e9 bf16 ~N(0, 0.02), each element independently (p=1e-3)
               multiplied by 8 (heavy-tail outliers).

The second argument of N(., .) is read as the standard deviation.
"""
from .generators import (  # noqa: F401
    bf16_bits_from_f32,
    bf16_bits_to_f32,
    normal_bf16,
    normal_bf16_rows,
    heavy_tail_chunk,
    keep_mask,
    CHUNK_ELEMS,
    n_chunks,
    linear_problem,
    linear_problem_rows,
    LinearProblem,
    WORKLOADS,
)
