"""World-size-2 data-parallel host logic on CPU (gloo): each rank computes the
adapter gradients of its own token shard (with the oracle, CPU only), writes
them into the flat gradient bucket the bench hands to the library, and one
all-reduce must reproduce the full-batch gradients."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_19_b200.dp import GradBucket, shard_tokens


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


SHAPES = [(24, 16, 8, 37), (40, 24, 16, 37)]       # (N, K, r, M_global)


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from oracle import linear as olin
    from synth import linear_problem
    bucket = GradBucket([(N, K, r) for (N, K, r, _) in SHAPES], "cpu", torch.float64)
    for (N, K, r, M), (dA, dB) in zip(SHAPES, bucket.views):
        p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=3)
        lo, hi = shard_tokens(M, world, rank)
        g = olin.lora_products(p.dY[lo:hi], p.X[lo:hi], p.A, p.B, p.s)
        dA.copy_(torch.from_numpy(g["dA"]))
        dB.copy_(torch.from_numpy(g["dB"]))
    bucket.allreduce_()
    if rank == 0:
        q.put(bucket.flat.numpy().copy())
    dist.barrier()
    dist.destroy_process_group()


def test_shard_tokens_partition():
    for M in (1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            parts = [shard_tokens(M, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [h - l for l, h in parts]
            assert max(sizes) - min(sizes) <= 1


def test_grad_bucket_views_are_contiguous_and_disjoint():
    b = GradBucket([(8, 4, 2), (16, 8, 4)], "cpu")
    ptrs = []
    for dA, dB in b.views:
        assert dA.is_contiguous() and dB.is_contiguous()
        ptrs.append((dA.data_ptr(), dA.numel()))
        ptrs.append((dB.data_ptr(), dB.numel()))
    assert sum(n for _, n in ptrs) == b.flat.numel()
    ptrs.sort()
    for (a, n), (c, _) in zip(ptrs, ptrs[1:]):
        assert a + 4 * n == c


def test_dp_allreduce_world2_matches_full_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    from oracle import linear as olin
    from synth import linear_problem
    ref = []
    for (N, K, r, M) in SHAPES:
        p = linear_problem(M, N, K, r, 2.0 * r, 0.02, seed=3)
        g = olin.lora_products(p.dY, p.X, p.A, p.B, p.s)
        ref += [g["dA"].ravel(), g["dB"].ravel()]
    np.testing.assert_allclose(got, np.concatenate(ref), rtol=1e-12, atol=1e-12)
