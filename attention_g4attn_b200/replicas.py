"""Multi-GPU plumbing of the benchmark: one independent replica of the hot path per rank.

The attention layer partitions into independent problems (sequences, kv heads), so N GPUs run N
replicas with no collective on the data path (weak scaling).  The only cross-rank traffic is the
timing: every rank's device-measured seconds are reduced with MAX, and the job rate counts the
units all ranks processed over that slowest time.
"""
from typing import List, Optional, Sequence


def max_over_ranks(seconds: Sequence[float], dist=None, device=None) -> List[float]:
    """Element-wise maximum of per-rank timings (a no-op without a process group)."""
    vals = [float(x) for x in seconds]
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return vals
    import torch
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(units_per_rank: float, seconds: float, world: int, scale: float = 1.0) -> float:
    """Whole-job throughput of `world` replicas that each processed `units_per_rank` units,
    over the slowest rank's time."""
    if seconds <= 0:
        raise ValueError("non-positive time")
    return world * units_per_rank / seconds / scale


def init_from_env(backend: str = "nccl", timeout_s: int = 120):
    """Initialise the process group from torchrun's environment; returns (dist, rank, world,
    local_rank) with dist None for a single process."""
    import os
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world <= 1:
        return None, 0, 1, 0
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist, rank, world, local_rank


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(n: int, argv: Sequence[str], port: Optional[int] = None,
                 timeout_s: Optional[float] = None, env: Optional[dict] = None) -> int:
    """Run `python argv...` as `n` local ranks under torch.distributed.run (rendezvous on
    127.0.0.1) and return its exit status.  The ranks inherit stdout / stderr, so the line
    rank 0 prints reaches the caller's stdout unchanged."""
    import os
    import subprocess
    import sys
    if n < 1:
        raise ValueError("need at least one rank")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=%d" % n, "--master-addr=127.0.0.1",
           "--master-port=%d" % (port or free_port())] + list(argv)
    e = dict(os.environ if env is None else env)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "LOCAL_WORLD_SIZE", "MASTER_ADDR",
              "MASTER_PORT", "GROUP_RANK", "ROLE_RANK", "TORCHELASTIC_RUN_ID"):
        e.pop(k, None)
    return subprocess.run(cmd, env=e, timeout=timeout_s).returncode
