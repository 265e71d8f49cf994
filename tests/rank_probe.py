"""Stand-in for one benchmark rank, for the launcher test on CPU (not collected by pytest).

Started by ``bench.launch_ranks`` under torchrun: it joins the process group the launcher set up
(gloo, CPU), takes the max over ranks of a rank-dependent time with ``bench.reduce_max`` and, on
rank 0 only, prints one JSON line with the world size -- the same shape of output that a real
benchmark rank prints.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402


def main():
    ws, rank, local = bench.dist_env()
    dist.init_process_group("gloo")
    try:
        mx = bench.reduce_max(1.0 + rank)
        if rank == 0:
            print(json.dumps({"n_gpus": ws, "max_seconds": mx, "argv": sys.argv[1:]}), flush=True)
    finally:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
