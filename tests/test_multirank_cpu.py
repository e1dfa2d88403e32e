"""The multi-process host path on CPU: two gloo ranks, as bench.py runs N GPUs
(one process each), check the block sharding and the max-over-ranks timing
reduction.  No GPU is touched."""
import os

import pytest
import torch.multiprocessing as mp

from trellis_coded_weight_tcq_b200.dist import block_range


def test_block_range_partitions_blocks():
    for n in (0, 1, 7, 229376):
        for world in (1, 2, 3, 8):
            ranges = [block_range(n, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        block_range(10, 2, 2)


def _worker(rank, world, port, out):
    import numpy as np
    import torch.distributed as dist

    from trellis_coded_weight_tcq_b200.dist import max_over_ranks, workload_for_rank

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workload_for_rank("tiny", rank)
        got = max_over_ranks([10.0 * rank + 1.0, -rank])
        digest = float(np.float64(wl.x.astype(np.float64).sum()))
        out.put((rank, got, digest, wl.x.shape))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, _, shape in res:
        assert got == [11.0, 0.0]          # max over ranks of (10 r + 1, -r)
        assert shape == (256, 64)
    assert res[0][2] != res[1][2]          # each rank encodes its own matrix (weak scaling)
