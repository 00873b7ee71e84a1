"""One rank of the two-rank host test of bench.py's multi-GPU logic (run under
torch.distributed.run with the gloo backend, no GPU)."""
import json
import os
import sys

import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def main():
    dist.init_process_group("gloo")
    rank, world = dist.get_rank(), dist.get_world_size()
    cpu = torch.device("cpu")
    # each rank reports a different elapsed time; all must agree on the slowest
    elapsed = 10.0 + 5.0 * rank
    slowest = bench.aggregate_max(elapsed, cpu)
    bench.barrier()
    value = bench.job_tokens_per_s(world, 4096, slowest / 100)
    out = {"rank": rank, "world": world, "slowest": slowest, "value": value}
    with open(os.path.join(sys.argv[1], f"rank{rank}.json"), "w") as f:
        json.dump(out, f)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
