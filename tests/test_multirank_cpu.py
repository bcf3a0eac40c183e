"""The multi-process side of bench.py on CPU: two gloo ranks over 127.0.0.1.

The decode path has no exchange between ranks (each rank advances its own
sequences); what the ranks share is the timing: the job takes as long as its
slowest rank, and the whole-job rate counts every rank's units over that time.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from linear_attention_recurrent_lq_b200 import inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out: dict):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup()
        # rank-dependent times: rank 1 is the slow one on the first entry
        mine = [10.0 + 5.0 * r, 7.0 - r, 3.0]
        got = bench.max_over_ranks(mine, torch, dist, w, "cpu")
        wl = bench.rank_workload(inputs.WORKLOADS["gdn_int8_b64h32"], r)
        out[r] = {"setup": (w, r, local), "max": got, "seed": wl.seed,
                  "rate": bench.whole_job_rate(1000, w, got[0])}
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_run_independent_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    for r in range(world):
        assert res[r]["setup"] == (world, r, r)
        # element-wise max over ranks, identical on every rank
        assert res[r]["max"] == [15.0, 7.0, 3.0]
        # 2 ranks x 1000 units over the slowest rank's 15 ms
        assert res[r]["rate"] == pytest.approx(2 * 1000 / 0.015)
    # each rank draws its own sequences (same shapes, different seed)
    assert res[0]["seed"] != res[1]["seed"]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2], torch, None, 1, "cpu") == [1.5, 2.0]
    wl = inputs.WORKLOADS["gdn_int8_b64h32"]
    assert bench.rank_workload(wl, 0) is wl
    assert bench.whole_job_rate(500, 1, 250.0) == pytest.approx(2000.0)
