"""Multi-rank host logic on CPU (gloo, world size 2): token-row sharding with no
data-path collective, and the max-over-ranks timing reduction the benchmark
uses.  The layer is row-independent (BitNet v2 write-up, section
"H-BitLinear": norm, transform and quantisation act per token), so the sharded
outputs concatenate to the unsharded output; the CPU oracle checks that."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from hadamard_rotated_int4_b200 import dist as hdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from hadamard_rotated_int4_b200 import inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X = inputs.activations("tiny")
        packed, alpha = oracle.pack_ternary(inputs.weights("tiny"))
        lo, hi = hdist.shard_rows(X.shape[0], world, rank)
        Y = oracle.hbitlinear_forward(X[lo:hi], packed, alpha, 4, threads=1)
        tmax = hdist.max_over_ranks(1.5 + rank)
        tsum = hdist.sum_over_ranks(1.0)
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi, Y))
        # the optional output gather (bf16 bit patterns widened to int32: the
        # gloo backend has no 16-bit integer type; NCCL takes bf16 directly)
        Yall = hdist.gather_rows(torch.from_numpy(Y.astype(np.int32)), X.shape[0])
        q.put((rank, tmax, tsum, gathered, Yall.numpy().astype(np.uint16)))
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_disjointly():
    for M in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [hdist.shard_rows(M, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        hdist.shard_rows(10, 2, 2)


def test_two_rank_gloo_sharded_layer_and_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from hadamard_rotated_int4_b200 import inputs

    X = inputs.activations("tiny")
    packed, alpha = oracle.pack_ternary(inputs.weights("tiny"))
    full = oracle.hbitlinear_forward(X, packed, alpha, 4, threads=1)
    for rank, tmax, tsum, gathered, Yall in results:
        assert tmax == 2.5 and tsum == 2.0
        Ycat = np.concatenate([g[2] for g in sorted(gathered, key=lambda g: g[0])])
        assert np.array_equal(Ycat, full)
        assert np.array_equal(Yall, full)  # the optional output all-gather
