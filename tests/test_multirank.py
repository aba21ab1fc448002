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
