"""One rank of the CPU (gloo) check of bench.py's multi-rank host logic; run by
test_bench_ranks.py with RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT set."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
# every rank times its own replica; the job's step time is the slowest rank's
mx = bench.max_over_ranks(100.0 + 7.0 * rank, device="cpu")
# the same collectives in the same order on every rank, also for a second figure
mx2 = bench.max_over_ranks(5.0 - rank, device="cpu")
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "max": mx, "max2": mx2, "prompt_tid": bench.prompt_tensor_id(rank)}))
