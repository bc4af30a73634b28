"""Multi-rank host logic on CPU: two gloo ranks (no GPU).

Sharding covers every block once, the reported step time is the maximum over ranks, and a
stack's bit allocation - the library's kronq_score_allocate run on every rank over the
all-reduced traces (pipeline.allocate_global) - is identical on both ranks and equal to the
oracle's allocation of all the traces in one process.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world_size, port, out):
    import torch.distributed as dist

    from post_quantization_b200 import dist as D
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world_size,
                            timeout=datetime.timedelta(seconds=60))
    try:
        n_blocks = 5
        mine = D.shard(n_blocks, rank, world_size)
        # a fake per-rank step time: the reported one must be the slowest rank's
        t = D.max_over_ranks(1.0 + rank)
        # traces of the 7 sublayers of each owned block (synthetic, deterministic)
        local = {}
        for b in mine:
            for s in range(7):
                i = b * 7 + s
                local[i] = (1.0 + 0.1 * i, 0.5 + ((i * 7919) % 13) / 3.0)
        from post_quantization_b200 import pipeline as P
        sizes = [4096 * 4096] * 4 + [11008 * 4096] * 3
        sizes = sizes * n_blocks
        # the library's allocation (host code of the C ABI) on the gathered traces
        _, bits = P.allocate_global(local, sizes, [2, 3, 4], 2.5)
        out[rank] = (mine, t, list(bits))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    (m0, t0, b0), (m1, t1, b1) = res[0], res[1]
    assert sorted(m0 + m1) == list(range(5)) and not set(m0) & set(m1)
    assert t0 == t1 == 2.0
    assert b0 == b1
    # same as one process over all blocks
    from oracle import kronq_oracle as O
    traces = [(1.0 + 0.1 * i, 0.5 + ((i * 7919) % 13) / 3.0) for i in range(35)]
    sizes = ([4096 * 4096] * 4 + [11008 * 4096] * 3) * 5
    assert O.score_allocate([a for a, _ in traces], [b for _, b in traces], sizes, [2, 3, 4],
                            2.5)[1] == b0


def test_shard_balanced():
    from post_quantization_b200.dist import shard
    for n in range(0, 40):
        for w in range(1, 9):
            parts = [shard(n, r, w) for r in range(w)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
