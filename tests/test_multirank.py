"""The N > 1 benchmark path on CPU: two gloo ranks exercise the same helpers
bench.py uses under torchrun (rank environment, per-rank seeds, max-over-ranks
step time, whole-job throughput).  The scan shards over independent batches,
so the only collectives are the timing ones tested here."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from mamba_ssd_scan_b200 import synthetic


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.rank_env()
        # each rank times a different step; the job's time is the slowest one
        local_ms = 1.0 + r
        ms = bench.max_over_ranks(local_ms, w, torch.device("cpu"))
        tokens = 4096
        value = bench.job_throughput(tokens, w, ms)
        seed = bench.rank_seed(1234, r)
        x = synthetic.make_fwd_inputs(1, 8, 2, 4, 4, 1, torch.float32, seed)["x"]
        out[r] = (r, w, local, ms, value, seed, float(x.sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        rank, w, local, ms, value, seed, xs = res[r]
        assert (rank, w, local) == (r, 2, r)
        assert ms == 2.0                          # max over ranks, seen by both
        assert value == pytest.approx(2 * 4096 / 2e-3)
    assert res[0][5] != res[1][5]                 # independent batches per rank
    assert res[0][6] != res[1][6]


def test_single_rank_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_throughput(100, 1, 10.0) == pytest.approx(1e4)


def test_bench_launches_its_own_ranks():
    """`bench.py --gpus 2` without a rank environment starts two ranks itself
    (here with the gloo plumbing only: no GPU on this host) and reports both."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--plumbing-only"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2
    assert sorted(rec["ranks_seen"]) == [0, 1]
    assert rec["ms_max_over_ranks"] == 2.0


def test_bench_rejects_a_mismatched_world():
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--plumbing-only"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode != 0
    assert "n_gpus" not in r.stdout
