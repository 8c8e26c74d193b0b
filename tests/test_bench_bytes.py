"""bench.py's roofline numerator and traffic lookup on the host: the algorithmic bytes of one
attention launch (every cached and new K/V row of each (request, KV head) once, queries read
and outputs written once) against a hand count and against the per-launch figures the
profiles record for two workloads, with the schedules rebuilt by the oracle; and the ncu
traffic entry, which holds only for the sources it was captured from."""
import numpy as np

import bench
import oracle
from oracle.schedule import lagged_round
from workloads import generate as G
from workloads.configs import CONFIGS, TINY


def test_attention_bytes_hand_count():
    cfg = TINY.with_(Hq=4, Hkv=2, D=8, dtype="bf16")
    # request 0: 64 cached keys and 2 draft tokens (3 verify tokens); request 1: empty cache,
    # no draft (1 verify token)
    kv_len, verify_len = [64, 0], [2, 0]
    kv_rows = (64 + 3) + (0 + 1)                    # per KV head, K and V each
    kv = kv_rows * cfg.Hkv * cfg.D * 2 * 2          # two KV heads, K and V, 2 bytes
    qo = (3 + 1) * cfg.Hq * cfg.D * 2 * 2           # queries in, outputs out
    assert bench.attn_bytes(kv_len, verify_len, cfg) == kv + qo
    f32 = cfg.with_(dtype="f32")
    assert bench.attn_bytes(kv_len, verify_len, f32) == 2 * (kv + qo)


def _schedule(name):
    """The scheduled verify lengths of a workload's benched round, rebuilt on the host with the
    generator's own draws (the order build_step_inputs takes them in) and the oracle."""
    cfg = CONFIGS[name]
    rng = np.random.default_rng(0)
    kv = G.kv_lengths(cfg, rng)
    G.page_table(kv, cfg.page_size, rng, reserve=cfg.K + 1)
    history = G.confidences(cfg, rng, 4)
    s = oracle.schedule_ref(history[lagged_round(3)], kv, G.step_time_table(cfg), cfg.T_cap)
    return cfg, kv, np.asarray(s["verify_len"])


def test_attention_bytes_match_the_recorded_workloads():
    cfg, kv, L = _schedule("qwen3-4b-64req")
    # every request verifies all five drafts: 6 tokens, 384 in all; per KV head and row,
    # 128 d x 2 B of K and of V
    assert np.all(L == 5)
    closed = int(np.sum((kv.astype(np.int64) + 6) * cfg.Hkv * 512)) + 384 * cfg.Hq * 512
    assert bench.attn_bytes(kv, L, cfg) == closed == 621_088_768
    cfg, kv, L = _schedule("lognormal-1024req")
    assert bench.attn_bytes(kv, L, cfg) == 22_324_592_640


def test_traffic_entry_holds_only_for_its_sources(monkeypatch):
    sha = bench.kernel_source_hash()
    monkeypatch.setitem(bench.NCU_TRAFFIC, "w", (sha, 1_010, 1_000))
    assert bench.measured_traffic("w", 1_000) == 1_010
    assert bench.measured_traffic("w", 2_000) == 2_020      # a smaller capture, scaled
    monkeypatch.setitem(bench.NCU_TRAFFIC, "w", ("0" * 40, 1_010, 1_000))
    assert bench.measured_traffic("w", 1_000) is None        # captured from other sources
    assert bench.measured_traffic("no-such-workload", 1_000) is None
    # the recorded entries are near the algorithmic bytes (no re-reads)
    for sha_, traffic, algo in bench.NCU_TRAFFIC.values():
        assert 1.0 <= traffic / algo < 1.05
