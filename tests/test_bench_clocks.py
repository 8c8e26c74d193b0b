"""bench.py's clock record on the host: parsing of the sampled nvidia-smi lines, which runs it
rejects (hardware or thermal slowdown, or an SM clock held low with no reason active; the power
cap alone is kept), and the one re-measurement, agreed by every rank so that all of them take
the same collective steps (two `gloo` ranks); and the strict lower bound on a step's logit bytes
(rows up to each request's first rejection)."""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = list(lines)
    return s.summary()


def test_summary_parses_nvidia_smi_lines():
    lines = ["1785, 1965, 980.12, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "1800, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "1770, 1965, 985.50, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "garbage line", ""]
    s = _sampler(lines)
    assert s == {"sm_mhz": 1785.0, "sm_max_mhz": 1965.0, "power_w": 985.5,
                 "reasons": ["sw_power_cap"], "samples": 3, "sufficient": False}
    assert _sampler([]) is None
    s = _sampler(["1500, 1965, 700, 0x8, Not Active, Active, Not Active, Not Active"])
    assert s["reasons"] == ["hw_thermal_slowdown"]


@pytest.mark.parametrize("summary,rejected", [
    (None, False),
    ({"sm_mhz": 1785.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}, False),
    ({"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}, False),
    ({"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": []}, False),
    ({"sm_mhz": 1200.0, "sm_max_mhz": 1965.0, "reasons": []}, True),     # leftover clock lock
    ({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown"]}, True),
    ({"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap", "sw_thermal_slowdown"]},
     True),
    ({"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["hw_thermal_slowdown"]}, True),
])
def test_clocks_rejected(summary, rejected):
    assert (bench.clocks_rejected(summary) is not None) == rejected


GOOD = {"sm_mhz": 1785.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 9}
BAD = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown"], "samples": 9}


def _fake_timed(records):
    calls = []

    def timed():
        calls.append(1)
        return len(calls), records[min(len(calls), len(records)) - 1]
    return timed, calls


def test_retry_single_rank():
    timed, calls = _fake_timed([GOOD])
    res, clocks = bench.measure_with_retry(timed, lambda f: f)
    assert (res, len(calls)) == (1, 1) and clocks == GOOD

    timed, calls = _fake_timed([BAD, GOOD])
    res, clocks = bench.measure_with_retry(timed, lambda f: f)
    assert (res, len(calls)) == (2, 2)                         # the second run is kept
    assert clocks["sm_mhz"] == GOOD["sm_mhz"]
    assert clocks["first_run"]["rejected"] == "hw_slowdown"

    timed, calls = _fake_timed([BAD, BAD])                      # measured again once only
    res, clocks = bench.measure_with_retry(timed, lambda f: f)
    assert (res, len(calls)) == (2, 2) and clocks["reasons"] == ["hw_slowdown"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _retry_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import torch
    timed, calls = _fake_timed([BAD, GOOD] if rank == 1 else [GOOD])
    res, clocks = bench.measure_with_retry(
        timed, lambda f: bench.agree_any(f, torch.device("cpu"), world))
    dist.barrier()           # both ranks reach the same collective steps
    out[rank] = (res, len(calls), clocks.get("first_run", {}).get("rejected"))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_retry_is_agreed_by_every_rank():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_retry_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    # rank 1 saw a slowdown: both ranks measured twice and kept the second run
    assert res[1] == (2, 2, "hw_slowdown")
    assert res[0] == (2, 2, "another rank's clock record")


def test_strict_lower_bound_counts_rows_up_to_the_first_rejection():
    from workloads.configs import TINY
    cfg = TINY.with_(V=10, dtype="bf16")
    L, a = [5, 0, 3], [2, 0, 3]
    # target rows 3 + 1 + 4, draft rows min(3, 5) + min(1, 0) + min(4, 3) = 3 + 0 + 3
    assert bench.logits_bytes_strict(L, a, cfg, greedy=False) == (8 + 6) * 10 * 2
    assert bench.logits_bytes_strict(L, a, cfg, greedy=True) == 8 * 10 * 2
    # every scheduled row: target 6 + 1 + 4, draft 5 + 0 + 3
    assert bench.logits_bytes(L, cfg, greedy=False) == (11 + 8) * 10 * 2
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(100):
        Lr = rng.integers(0, 6, size=16)
        ar = rng.integers(0, Lr + 1)
        for g in (False, True):
            assert bench.logits_bytes_strict(Lr, ar, cfg, g) <= bench.logits_bytes(Lr, cfg, g)
            if not g and np.all(ar == Lr):
                # all accepted: every draft row plus one extra target row per request is read
                assert bench.logits_bytes_strict(Lr, ar, cfg, g) == bench.logits_bytes(Lr, cfg, g)
