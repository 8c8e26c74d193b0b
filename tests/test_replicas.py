"""Multi-replica host logic on CPU: two `gloo` ranks, as `bench.py --gpus N` runs them.

The verify step shards by request with no data-path collective; the only cross-rank steps are
the reduction of timings (max over ranks) and token counts (sum), and the barrier around the
timed region.  These tests run that logic with world size 2 on the host, including a rank that
leaves before the collective (the survivor must fail within the process-group timeout rather
than wait for ever).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from oracle.schedule import lagged_round
from workloads.configs import TINY
from workloads.generate import build_step_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _replica_worker(rank, world, port, out):
    _init(rank, world, port, 60)
    # each replica schedules its own batch (seed = rank) with the oracle
    inp = build_step_inputs(TINY, "cpu", seed=rank, layers=1)
    conf = inp.conf_history[lagged_round(inp.round_idx)]
    L = oracle.schedule_ref(conf, inp.kv_len.numpy(), inp.t_ms.numpy(), TINY.T_cap)["verify_len"]
    ms = 1.0 + rank           # rank 1 is the slower replica
    agg = bench.reduce_replicas(ms, 0.5 * (rank + 1), 2.0 * (rank + 1), int(np.sum(L)),
                                rank + 1, TINY.R, world, torch.device("cpu"))
    dist.barrier()
    out[rank] = (agg, int(np.sum(L)))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_replicas_reduce_max_time_and_sum_tokens():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_replica_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    L0, L1 = res[0][1], res[1][1]
    for rank in range(world):
        agg = res[rank][0]
        assert agg["ms_step"] == 2.0 and agg["attn_ms"] == 1.0 and agg["e2e_ms"] == 4.0
        assert agg["L_tot"] == L0 + L1 and agg["acc_tot"] == 3 and agg["R_tot"] == 2 * TINY.R
    # the job's value is the sum of every replica's tokens over the slowest replica's time
    assert res[0][0]["L_tot"] / res[0][0]["ms_step"] == (L0 + L1) / 2.0


def test_replicas_draw_distinct_batches():
    a = build_step_inputs(TINY, "cpu", seed=0, layers=1)
    b = build_step_inputs(TINY, "cpu", seed=1, layers=1)
    assert not torch.equal(a.q, b.q) and not torch.equal(a.kv_len, b.kv_len)


def _leaving_worker(rank, world, port, out):
    _init(rank, world, port, 5)
    if rank == 1:
        # a replica that fails on the host before the reduction and leaves
        out[rank] = "left"
        os._exit(0)
    try:
        bench.reduce_replicas(1.0, 1.0, 1.0, 1, 1, 1, world, torch.device("cpu"))
        out[rank] = "completed"
    except Exception as e:  # the collective ends with an error instead of waiting for ever
        out[rank] = "error:" + type(e).__name__
    os._exit(0)


@pytest.mark.timeout(180)
def test_rank_leaving_before_collective_fails_the_survivor_quickly():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        ctx = mp.get_context("spawn")
        port = _free_port()
        procs = [ctx.Process(target=_leaving_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert res.get(1) == "left"
    assert str(res.get(0, "")).startswith("error:"), res
