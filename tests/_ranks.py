"""Rank bodies for the multi-process tests (imported by spawned children, so
they live in a module of their own)."""
import datetime
import os


def reduction_rank(rank, world, port, out):
    """One gloo rank: reads its environment the way bench.py does, reduces a
    rank-dependent time and work, and reports what it saw."""
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        env = bench._rank_env()
        ms, work = bench._reduce_max_sum(10.0 + 5.0 * rank, 100.0 * (rank + 1), "cpu")
        out.put((rank, env, ms, work, bench._rank_seed(7, rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()
