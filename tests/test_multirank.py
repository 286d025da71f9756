"""World-size-2 runs of the bench's multi-rank host logic on CPU (gloo): every rank gets a cache
of the same shape with its own data (weak scaling, no data-path collective), the job's time is
the slowest rank's, the reported rate counts the bytes of all ranks, and the reference arm runs
on rank 0 only."""
import contextlib
import datetime
import io
import json
import os
import socket
import sys
import types

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from random_access_kv_fq_b200 import workloads as wl
        cache = bench.rank_cache(wl.GPT2, rank)
        x = wl.slab(cache, "K", 0, 0)
        ms = bench.max_over_ranks(torch, dist, 10.0 * (rank + 1), torch.device("cpu"))
        rate = bench.whole_job_rate(world, 1.5e9, 4, ms)
        info = {"rank": rank, "n": cache.n, "d": cache.d, "seed": cache.seed,
                "checksum": float(np.asarray(x, dtype=np.float64).sum()), "ms": ms, "rate": rate}
        gathered = [None] * world
        dist.all_gather_object(gathered, info)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(gathered, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_host_logic(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2,
                       start_method="spawn")
    views = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert views[0] == views[1]  # both ranks saw the same gathered picture
    r0, r1 = views[0]
    assert (r0["n"], r0["d"]) == (r1["n"], r1["d"])           # same shape per rank
    assert r0["seed"] != r1["seed"]                           # its own data
    assert r0["checksum"] != r1["checksum"]
    assert r0["ms"] == r1["ms"] == 20.0                       # the slowest rank's time
    assert abs(r0["rate"] - 2 * 1.5e9 * 4 / 0.020 / 1e9) < 1e-9  # bytes of both ranks


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = types.SimpleNamespace(workload="gpt2", tokens=None, steps=1, warmup=0)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(args)
    assert out.getvalue() == ""
