"""Worker of tests/test_multirank.py: one rank of the benchmark's host-side
multi-rank logic (process group, barrier, max over ranks) on gloo."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    world, rank, local = bench.dist_setup()
    bench.barrier(world)
    m = bench.max_over_ranks(1.5 + rank, world)
    bench.barrier(world)
    print(f"rank {rank} of {world}: max {m}", flush=True)
    import torch.distributed as dist
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
