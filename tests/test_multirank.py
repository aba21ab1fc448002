"""The multi-GPU path of the benchmark on CPU: two gloo ranks.

The codec shards by whole tensors (ranks are independent replicas), so the only cross-rank steps
are the barrier and the max-over-ranks timing; the whole-job value is weak-scaling throughput.
"""
import os
import socket
import tempfile

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, outdir):
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(1.0 + 0.5 * rank, "cpu")   # rank 1 is the slow one
        dist.barrier()
        value = bench.weak_scaling_value(10 ** 9, world, ms)
        with open(os.path.join(outdir, f"r{rank}"), "w") as f:
            f.write(f"{ms} {value}")
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank, args=(world, _free_port(), d), nprocs=world, join=True)
        res = [tuple(map(float, open(os.path.join(d, f"r{r}")).read().split())) for r in range(world)]
    for ms, value in res:
        assert ms == 1.5                                 # max over ranks, identical on every rank
        assert abs(value - 2 * 1e9 / 1.5e-3 / 1e9) < 1e-9  # 2 replicas x 1 GB in 1.5 ms


def _rank_encode(rank, world, port, outdir):
    """Each rank encodes its own row range of one weight with the oracle (no data exchange); the
    ranks then all-gather their per-chunk word counts, the one integer per chunk a concatenated
    stream would need to place every shard."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from post_quantization_tile_b200 import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = W.llama_weight(4096, 4096, seed=1)[:192, :512]
        per = x.shape[0] // world                                   # 96 rows: whole 32-row chunks
        mine = np.ascontiguousarray(x[rank * per:(rank + 1) * per])
        code = oracle.encode(mine, 128, oracle.E8, 0.3, 7)
        counts = torch.from_numpy(np.diff(code.chunk_word.astype(np.int64)))
        gathered = [torch.zeros_like(counts) for _ in range(world)]
        dist.all_gather(gathered, counts)
        if rank == 0:
            np.save(os.path.join(outdir, "gathered.npy"), torch.stack(gathered).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_row_shards_give_the_single_process_chunks():
    """Row-range sharding is exact: every chunk of the single-process code has the word count that
    the rank owning its rows computed alone."""
    import numpy as np

    import oracle
    from post_quantization_tile_b200 import workloads as W
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_encode, args=(world, _free_port(), d), nprocs=world, join=True)
        g = np.load(os.path.join(d, "gathered.npy"))               # [rank, tile column * 3 chunks]
    x = W.llama_weight(4096, 4096, seed=1)[:192, :512]
    whole = oracle.encode(np.ascontiguousarray(x), 128, oracle.E8, 0.3, 7)
    counts = np.diff(whole.chunk_word.astype(np.int64)).reshape(4, 6)  # tile column x row chunk
    per_rank = g.reshape(world, 4, 3)
    np.testing.assert_array_equal(counts, np.concatenate([per_rank[0], per_rank[1]], axis=1))
