"""The N > 1 bench path on CPU: two gloo ranks run the replicas' bookkeeping -- rank-specific
rows, the max over ranks of the timed region, whole-job throughput -- with no data exchanged
between the replicas' drafts."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import bench
    from draft_block_causal_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        wl = bench.rank_workload(rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, wl["input_seed"])
        # each replica drafts its own rows: a small head with this rank's input seed
        small = dict(wl, B=1, L=4, d=64, Hs=32, r=16, V=1000, dtype=synth.F32, name="tiny-rank")
        data = synth.make_workload(small)
        sums = [None] * world
        dist.all_gather_object(sums, float(abs(data["hidden"]).sum()))
        local_ms = 10.0 + 5.0 * rank  # the replicas' timed regions differ
        total = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_throughput(wl["B"], world, 4, total)
        if rank == 0:
            with open(out_path, "w") as f:
                json.dump({"seeds": seeds, "sums": sums, "total": total, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_replicas(tmp_path):
    out = str(tmp_path / "r.json")
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    r = json.load(open(out))
    assert len(set(r["seeds"])) == 2          # rank-specific rows
    assert r["sums"][0] != r["sums"][1]        # the replicas' inputs differ
    assert r["total"] == 15.0                  # the slowest replica's time, on every rank
    assert r["value"] == pytest.approx(1 * 2 * 4 / 15e-3)  # whole-job throughput over both replicas


def test_single_process_bookkeeping():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, None, "cpu") == 12.5
    assert bench.job_throughput(32, 1, 10, 100.0) == pytest.approx(3200.0)
