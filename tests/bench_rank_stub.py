"""One rank of a CPU (gloo) run of bench.py's launcher and rank plumbing, for
tests/test_multirank.py: bench.run_ranks with an arm that stands in for the device arms.
Each rank times its own replica (rank r: 10 + 5 r ms); the arm takes the slowest rank's
time and the whole-job rates with the same helpers as the device arms."""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def stub_arm(args, rank, world, local_rank):
    import torch
    dist = None
    if world > 1:
        import torch.distributed as dist
    ms = bench.reduce_max(10.0 + 5.0 * rank, dist, torch.device("cpu"))
    value, tokens_per_s = bench.weak_scaling_rates(1e9, 64, world, ms)
    return {"n_gpus": world, "value": value, "tokens_per_s": tokens_per_s, "ms_per_step": ms,
            "rank": rank, "local_rank": local_rank}


if __name__ == "__main__":
    args = bench.parse_args(sys.argv[1:])
    res = bench.run_ranks(args, stub_arm, backend="gloo")
    if res is not None:
        print(json.dumps(res), flush=True)
