"""The bench's N > 1 host path on CPU: world_size-2 gloo ranks.

Each rank runs its own replica of the MoE layer (its own batch and routing,
weak scaling); the only cross-rank steps are the max of the per-rank times and
the whole-job rate, plus the reference arm printing on rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import synthetic
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank_ms = 10.0 + 7.0 * rank                       # rank 1 is the slower one
        slowest = bench.max_over_ranks(per_rank_ms, world, "cpu")
        rate = bench.whole_job_rate(2.0e12, world, 5, slowest)
        # each rank's replica routes its own batch (seed = rank)
        r = synthetic.route_topk_softmax(rank, 256, 32, 4)
        digest = int(np.asarray(r["row_index"], dtype=np.int64)[:64].sum())
        dist.barrier()
        with open(f"{out_path}.{rank}", "w") as f:
            json.dump({"slowest": slowest, "rate": rate, "digest": digest}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_rate(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    out = str(tmp_path / "rank")
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    res = [json.load(open(f"{out}.{r}")) for r in range(world)]
    # every rank sees the slowest rank's time; the rate counts all ranks' work
    assert res[0]["slowest"] == res[1]["slowest"] == 17.0
    assert res[0]["rate"] == pytest.approx(world * 2.0e12 * 5 / 17.0e-3)
    # replicas are independent batches
    assert res[0]["digest"] != res[1]["digest"]


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1e9, 1, 4, 2.0) == pytest.approx(2e12)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
                        "--experts", "16", "--tokens", "256"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    if rank == 0:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
