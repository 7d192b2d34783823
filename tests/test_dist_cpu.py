"""The N > 1 plumbing of bench.py on two CPU ranks over gloo: the process group,
the max-over-ranks step time, the whole-job throughput, per-rank input sets that do
not overlap (weak scaling, no collective on the data path), and the reference arm
doing its work on rank 0 alone."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout
from types import SimpleNamespace

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    from workloads import WORKLOAD_NAMES, make_workload
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(w, local, "gloo")
    res = {}
    # each rank timed a different total; the job's step time is the slowest rank's
    ms_local = [8.0, 12.0][rank]
    res["ms_per_step"], res["tokens_s"] = bench.job_time_and_throughput(ms_local, 4, 256, w, dist)
    # the rank's own tiny batch: its inputs come from its own seed
    idx = WORKLOAD_NAMES.index("tiny_sgmv")
    wl = make_workload(idx, device="cpu", seed=bench.rank_seed(idx, rank, 0))
    x = wl.calls[0].X.float()
    res["x_sum"] = float(x.sum())
    # gather the per-rank sums (test only) to compare the batches across ranks
    t = torch.tensor([res["x_sum"]], dtype=torch.float64)
    gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(w)]
    dist.all_gather(gathered, t)
    res["x_sums"] = [float(g.item()) for g in gathered]
    dist.barrier()
    dist.destroy_process_group()
    # reference arm: rank != 0 returns at once without output
    if rank != 0:
        buf = io.StringIO()
        args = SimpleNamespace(workload="tiny_sgmv", steps=1, warmup=0, reference_seconds=1.0)
        with redirect_stdout(buf):
            bench.run_reference(args)
        res["reference_output"] = buf.getvalue()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r0 = json.loads((tmp_path / "r0.json").read_text())
    r1 = json.loads((tmp_path / "r1.json").read_text())
    # max over ranks: 12 ms / 4 steps; 2 ranks x 256 tokens per step in that time
    for r in (r0, r1):
        assert r["ms_per_step"] == pytest.approx(3.0)
        assert r["tokens_s"] == pytest.approx(2 * 256 / 3e-3)
    # independent batches: the two ranks' inputs differ, and both ranks saw both sums
    assert r0["x_sums"] == r1["x_sums"]
    assert r0["x_sums"][0] != r0["x_sums"][1]
    assert r1["reference_output"] == ""


def test_rank_seeds_do_not_overlap():
    sys.path.insert(0, ROOT)
    import bench
    seeds = {bench.rank_seed(i, r, s) for i in range(5) for r in range(8) for s in range(16)}
    assert len(seeds) == 5 * 8 * 16
