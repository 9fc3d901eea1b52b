"""The N > 1 path of the benchmark on CPU: two gloo ranks, each an independent replica, reduce
their timings with MAX and report the whole-job rate (no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from attention_g4attn_b200 import replicas
    dist, r, w, lr = replicas.init_from_env("gloo", timeout_s=30)
    try:
        # rank-dependent device times: rank 1 is the slowest on the first value only
        local = [1.0 + r, 5.0 - r, 0.25]
        got = replicas.max_over_ranks(local, dist)
        rate = replicas.job_rate(100.0, got[0], w)
        q.put((r, w, got, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_reduce_timings_with_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, got, rate in res:
        assert w == 2
        assert got == [2.0, 5.0, 0.25]          # max over ranks, element-wise
        assert rate == pytest.approx(2 * 100.0 / 2.0)   # all ranks' units over the slowest time


def test_single_process_is_a_no_op():
    from attention_g4attn_b200 import replicas
    assert replicas.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert replicas.job_rate(10.0, 2.0, 1) == 5.0
    with pytest.raises(ValueError):
        replicas.job_rate(1.0, 0.0, 1)


def test_launcher_runs_n_ranks(tmp_path):
    """bench.py --gpus N started without torchrun re-launches itself through
    replicas.launch_ranks: N local ranks under torch.distributed.run, rendezvous on
    127.0.0.1.  Here with 2 gloo ranks of a small child script on CPU."""
    import json
    from attention_g4attn_b200 import replicas
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "replica_child.py")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    rc = replicas.launch_ranks(2, [child, str(tmp_path)], timeout_s=240, env=env)
    assert rc == 0
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(2)]
    for r, x in enumerate(res):
        assert x["rank"] == r and x["world"] == 2 and x["local_rank"] == r
        assert x["master"] == "127.0.0.1"
        assert x["got"] == [2.0, 3.0]
        assert x["rate"] == pytest.approx(2 * 10.0 / 2.0)


def test_bench_refuses_a_rank_count_that_disagrees_with_gpus():
    """Under torchrun, bench.py checks that WORLD_SIZE equals --gpus before any GPU work."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "4"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 2
    assert "WORLD_SIZE=2" in r.stderr
