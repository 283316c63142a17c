"""Multi-process logic on CPU (gloo, world size 2): row sharding covers every
row exactly once, per-rank results gathered in rank order equal the
single-process result, and the timing reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from prng_seeded_decompress_b200 import dist_util, inputs


def test_row_shard_partitions_rows():
    for rows in (0, 1, 7, 8192, 57344):
        for world in (1, 2, 3, 8):
            spans = [dist_util.row_shard(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(e - s for s, e in spans) - min(e - s for s, e in spans) <= 1
    with pytest.raises(ValueError):
        dist_util.row_shard(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        L = inputs.make_layer(37, 203, 12, 4, seed=5)
        _, x = inputs.make_activations((203,), "f16", 6)
        r0, r1 = dist_util.row_shard(37, world, rank)
        fmt, rec, ep = dist_util.shard_view(L["fmt"], L["rec"], L["eplane"], r0, r1)
        y, _ = oracle.gemv(fmt, rec, ep, x)
        # variable-size gather: pad to the largest shard
        n = torch.tensor([r1 - r0])
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, n)
        m = max(int(s) for s in sizes)
        buf = torch.zeros(m, dtype=torch.float64)
        buf[: r1 - r0] = torch.from_numpy(y)
        parts = [torch.zeros(m, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts, buf)
        full = torch.cat([p[: int(s)] for p, s in zip(parts, sizes)]).numpy()
        t = dist_util.max_over_ranks(1.5 + rank)
        if rank == 0:
            ref, _ = oracle.gemv(L["fmt"], L["rec"], L["eplane"], x)
            result_q.put((bool(np.array_equal(full, ref)), t))
    finally:
        dist.destroy_process_group()


def test_sharded_gemv_gathers_to_full_result_gloo():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    same, t = q.get(timeout=10)
    assert same and t == 2.5
