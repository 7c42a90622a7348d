"""Worker of tests/test_multirank.py (a module of its own so spawned
processes can import it)."""
import datetime
import os


def run(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [12.0, 15.5, 9.25, 14.0][rank]
        slowest = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(world, 64, 10, slowest)
        queue.put((rank, slowest, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()
