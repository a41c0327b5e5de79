"""Splitting one causal convolution over ranks (the multi-GPU path), on CPU.

Host logic only: which rows a rank owns, its contiguous slab, and the optional
all-gather.  Under two gloo ranks each rank convolves its slab of one seeded
tensor -- with the oracle, standing in for the single-GPU call -- the slabs
are gathered, and the result must equal the unsharded oracle bit for bit
(rows are independent, so a partition changes no sum).
"""
import os
import socket

import numpy as np
import pytest

from spectral_sequence_mixing_b200 import partition

CASES = [
    # (B, L, D, dtype): B = 1 splits channels (long-context shape), B >= world splits batches
    (1, 64, 10, "f32"),
    (1, 33, 3, "f32"),
    (3, 40, 6, "f32"),
    (4, 24, 5, "i32"),
    (1, 1, 1, "f32"),  # fewer channels than ranks: rank 1 owns no rows
]


def test_shards_cover_every_row_once():
    for B in (1, 2, 3, 7, 8):
        for D in (1, 2, 5, 768, 1024):
            for world in (1, 2, 3, 4, 8):
                owner = np.zeros((B, D), np.int64)
                for rank in range(world):
                    s = partition.shard_for(B, D, world, rank)
                    assert s.axis == ("B" if B >= world else "D")
                    owner[s.b0:s.b1, s.d0:s.d1] += 1
                    nb, nd = s.shape_bd
                    # balanced: slabs differ by at most one batch / channel
                    if s.axis == "B":
                        assert nd == D and abs(nb - B / world) < 1
                    else:
                        assert nb == B and abs(nd - D / world) < 1
                assert (owner == 1).all(), (B, D, world)


def test_take_and_place_roundtrip():
    rng = np.random.Generator(np.random.PCG64(7))
    x = rng.standard_normal((1, 9, 10)).astype(np.float32)
    full = np.zeros_like(x)
    for rank in range(3):
        s = partition.shard_for(1, 10, 3, rank)
        part = partition.take(x, s)
        assert part.flags["C_CONTIGUOUS"] and part.shape == (1, 9, s.d1 - s.d0)
        partition.place(full, part, s)
    assert np.array_equal(full, x)


def test_bad_arguments():
    with pytest.raises(ValueError):
        partition.shard_for(1, 4, 2, 2)
    with pytest.raises(ValueError):
        partition.shard_for(0, 4, 2, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, L, D, dtype, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    if dtype == "i32":
        return (rng.integers(-128, 128, (B, L, D)).astype(np.int32),
                rng.integers(-128, 128, (B, L, D)).astype(np.int32))
    return rng.standard_normal((B, L, D)).astype(np.float32), rng.standard_normal((B, L, D)).astype(np.float32)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    results = []
    for i, (B, L, D, dtype) in enumerate(CASES):
        v, g = _inputs(B, L, D, dtype, 100 + i)  # every rank draws the same global tensor
        s = partition.shard_for(B, D, world, rank)
        vl, gl = partition.take(v, s), partition.take(g, s)
        if vl.size:
            rl = oracle.causal_conv_int(vl, gl) if dtype == "i32" else oracle.causal_conv(vl, gl)[0]
        else:
            rl = np.zeros(vl.shape, np.int64 if dtype == "i32" else np.float64)
        full = partition.gather(torch.from_numpy(rl), B, L, D, world, rank)
        if rank == 0:
            ref = oracle.causal_conv_int(v, g) if dtype == "i32" else oracle.causal_conv(v, g)[0]
            results.append((i, s.axis, bool(np.array_equal(full.numpy(), ref))))
    q.put((rank, results))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_partition_one_tensor():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert len(out[0]) == len(CASES)
    for i, axis, same in out[0]:
        B, L, D, dtype = CASES[i]
        assert axis == ("B" if B >= 2 else "D")
        assert same, f"sharded result differs from the unsharded oracle for {CASES[i]}"
