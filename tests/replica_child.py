"""One rank of the launcher test (tests/test_replicas_gloo.py): joins the gloo group that
torch.distributed.run set up, reduces a rank-dependent timing with MAX and writes what it
saw to <out_dir>/rank<r>.json."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from attention_g4attn_b200 import replicas  # noqa: E402


def main():
    out_dir = sys.argv[1]
    dist, rank, world, local_rank = replicas.init_from_env("gloo", timeout_s=60)
    try:
        got = replicas.max_over_ranks([1.0 + rank, 3.0 - rank], dist)
        rate = replicas.job_rate(10.0, got[0], world)
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"rank": rank, "world": world, "local_rank": local_rank,
                       "master": os.environ.get("MASTER_ADDR"), "got": got, "rate": rate}, f)
        if dist:
            dist.barrier()
    finally:
        if dist:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
