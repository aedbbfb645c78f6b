"""The multi-GPU path on CPU: two `gloo` ranks in separate processes.

The path does not shard (each rank runs an independent replica stream, no
data-path collective), so what N > 1 adds is host logic: per-rank replica
seeds, the max-over-ranks time and the whole-job rate. These run here with
the same functions bench.py uses, and each rank drives its own replica's page
state through the library (host-only plans, no GPU).
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    import workload
    import paged_kv_cache_frame_b200 as pkv

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # timing: every rank gets the slowest rank's time
        ms = 100.0 + 50.0 * rank
        ms_max = bench.max_over_ranks(ms, world)
        rate = bench.whole_job_rate(320, world, ms_max)
        # each rank's replica: its own seed, keyframe draw and page state
        wl = workload.WORKLOADS[2]
        seed = bench.replica_seed(1, rank)
        keep = workload.keyframe_mask(wl, seed, n_frames=40)
        c = pkv.PagedKVCache(wl.max_pages, wl.page_size, wl.H, wl.D, wl.S, wl.W, num_blocks=2)
        for f in range(40):
            c.defer_eviction(True)
            for b in range(2):
                c.append_frame(b, None, None)
            c.evict_frames()
            table, lpl = pkv.Plan([c]).page_table()
            if keep[f]:
                c.commit_frame()
            else:
                c.rollback_last_frame()
        stats = c.get_stats()
        got = [None] * world
        dist.all_gather_object(got, {"ms_max": ms_max, "rate": rate, "seed": seed, "keep": keep.tolist(),
                                     "stats": stats, "table": table, "lpl": lpl})
        if rank == 0:
            torch.save(got, os.path.join(out_dir, "ranks.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_replica_streams(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(tmp_path / "ranks.pt")
    # the slowest rank's time, seen by every rank
    assert [g["ms_max"] for g in got] == [150.0, 150.0]
    # whole-job rate: frames of all ranks over the slowest time
    assert got[0]["rate"] == pytest.approx(2 * 320 / 0.150)
    # independent replicas: different seeds and keyframe draws ...
    assert got[0]["seed"] != got[1]["seed"]
    assert got[0]["keep"] != got[1]["keep"]
    # ... each with a consistent page state: committed frames = kept frames
    for g in got:
        assert g["stats"]["frame_count"] == int(np.sum(g["keep"]))
        assert 1 <= g["lpl"] <= 256
        assert len(set(g["table"])) == len(g["table"])
