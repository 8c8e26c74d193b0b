"""Benchmark of one DSpark confidence-scheduled verify step on B200.

A step = dspark_schedule + dspark_verify_attn_plan + `layers` x dspark_verify_attn + dspark_accept
over one batch of seeded synthetic inputs already resident in HBM.  Metric: verified draft
tokens/s per verify step (sum of scheduled verify lengths / step time), plus accepted and
emitted tokens/s and the achieved HBM bandwidth of the step and of its dominant kernel.
The timed region is one replay of the K steps captured as a CUDA graph (the library sizes every
launch by capacity, so consecutive steps need no host involvement); the eager step time is
reported beside it.  After timing, the step's schedule and every request's acceptance are
checked against the float64 oracle, and sampled attention rows of the last layer call; the
line reports the decisions the oracle flags as within 1e-6 of a threshold.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dspark|reference]
                    [--workload lognormal-1024req] [--layers 36]
    python bench.py --report [--report-md FILE]    # every workload, one JSON line each

Multi-GPU runs (torchrun, one process per GPU) are independent replicas: each rank verifies its
own request batch (seed = rank) with no data-path collective; the step time is the max over
ranks and `value` sums every rank's tokens.  `--impl reference` times the float64 CPU oracle
on the host cores, on the same bounded sample of the same workload that the `cpu_baseline`
leg of the default run times (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads.configs import CONFIGS, SWEEP_LEVELS  # noqa: E402
from workloads.generate import build_step_inputs, flatten_target  # noqa: E402

METRIC = "verified draft tokens/s per verify step (1 B200); achieved HBM GB/s vs peak"
UNIT = "tokens/s"
# the largest single-GPU workload the 70%-of-roofline target names (1024 requests, lognormal
# KV lengths up to 32 768, 64/8 heads, V 129 280, T = 0.7)
DEFAULT_WORKLOAD = "lognormal-1024req"
REPORT_WORKLOADS = (["qwen3-4b-64req", "mixed-256req", "lognormal-1024req",
                     "lognormal-1024req-greedy"] + [f"sweep-{R}req" for R in SWEEP_LEVELS])
MIN_CLOCK_SAMPLES = 10


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # start timing only once the sampler is producing (nvidia-smi takes a while to start)
            t_end = time.time() + 10.0
            while not self.lines and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.02)
            self.lines.clear()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[2]))
            except ValueError:
                pass
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "power_w": statistics.median(pw) if pw else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "sufficient": len(sm) >= MIN_CLOCK_SAMPLES}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch, from an ncu
# capture, keyed by the SHA-1 of the sources the attention kernel is built from (ATTN_SOURCES);
# any change to those voids the figure.  Entries: (sha, bytes, algorithmic bytes of the capture);
# a capture of another size of the same workload is scaled by algorithmic bytes.
NCU_TRAFFIC = {
    # one launch of the full workload (a 1-pass capture): 22 410 693 632 B read + 37 202 176 B
    # written, 22 324 592 640 algorithmic bytes
    "lognormal-1024req": ("e840b321bde13108a61c6304d457b563a463b647", 22447895808, 22324592640),
    "lognormal-1024req-greedy": ("e840b321bde13108a61c6304d457b563a463b647", 22447895808,
                                 22324592640),
    # 626 555 904 B read + 4 280 064 B written, 621 088 768 algorithmic bytes
    "qwen3-4b-64req": ("e840b321bde13108a61c6304d457b563a463b647", 630835968, 621088768),
}

ATTN_SOURCES = ("attn_tk.cuh", "attn_common.cuh", "ptx_sm100.cuh", "common.cuh", "dspark.cu")


def kernel_source_hash():
    import hashlib
    d = os.path.join(ROOT, "speculative_decoding_verification_survival_b200", "csrc")
    h = hashlib.sha1()
    for name in ATTN_SOURCES:
        with open(os.path.join(d, name), "rb") as fh:
            h.update(name.encode() + b"\0" + fh.read())
    return h.hexdigest()


def measured_traffic(workload, algorithmic_bytes):
    """ncu DRAM bytes of one launch of this workload, or None when the kernel sources changed
    since the capture; a capture of a smaller case is scaled by algorithmic bytes."""
    rec = NCU_TRAFFIC.get(workload)
    if rec is None or rec[0] != kernel_source_hash():
        return None
    return int(round(rec[1] * algorithmic_bytes / rec[2]))


def attn_bytes(kv_len, verify_len, cfg):
    """Algorithmic bytes of one attention launch: every cached and new K/V row of every
    (request, KV head) once, queries read once, outputs written once."""
    esz = 2 if cfg.dtype == "bf16" else 4
    n = np.asarray(kv_len, np.int64)
    Q = 1 + np.asarray(verify_len, np.int64)
    T = int(Q.sum())
    kv = int(((n + Q) * cfg.Hkv * cfg.D * 2 * esz).sum())
    return kv + 2 * T * cfg.Hq * cfg.D * esz


def logits_bytes(verify_len, cfg, greedy):
    esz = 2 if cfg.dtype == "bf16" else 4
    L = np.asarray(verify_len, np.int64)
    rows = int((1 + L).sum()) + (0 if greedy else int(L.sum()))
    return rows * cfg.V * esz


def logits_bytes_strict(verify_len, accepted_len, cfg, greedy):
    """The logit bytes a step must read at the least: per request the target rows of positions
    1..a+1 and, unless greedy, the draft rows of positions 1..min(a+1, L), i.e. the rows up to
    and including the first rejection (or the bonus row); the rest of the block is never used."""
    esz = 2 if cfg.dtype == "bf16" else 4
    L = np.asarray(verify_len, np.int64)
    a = np.asarray(accepted_len, np.int64)
    rows = int((a + 1).sum()) + (0 if greedy else int(np.minimum(a + 1, L).sum()))
    return rows * cfg.V * esz


REJECT_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(summary):
    """Why a timed run's clock record rejects it, or None when it stands.  A run is rejected
    when it saw a hardware or thermal slowdown, or when its SM clock stayed well below the
    maximum with no reason active (a leftover clock lock).  sw_power_cap alone is kept."""
    if not summary or "sm_mhz" not in summary:
        return None
    bad = [r for r in summary.get("reasons", []) if r in REJECT_REASONS]
    if bad:
        return "+".join(bad)
    if not summary.get("reasons") and summary["sm_mhz"] < 0.75 * summary["sm_max_mhz"]:
        return "SM clock held below 0.75 of max with no reason active"
    return None


def agree_any(flag, device, world):
    """True on every rank when `flag` is true on any rank (so that all ranks take the same
    collective steps)."""
    if world == 1:
        return bool(flag)
    t = torch.tensor([int(bool(flag))], dtype=torch.int32, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return bool(t.item())


def measure_with_retry(timed, agree):
    """timed() -> (result, clocks).  When the clock record of the run rejects it on any rank,
    every rank measures once more and keeps the second result; the first run's clocks and the
    reason are kept under clocks["first_run"]."""
    res, clocks = timed()
    why = clocks_rejected(clocks)
    if agree(why is not None):
        first = dict(clocks or {}, rejected=why or "another rank's clock record")
        res, clocks = timed()
        clocks = dict(clocks, first_run=first) if clocks else {"first_run": first}
    return res, clocks


def kv_copies_for(cfg, kv_bytes_per_layer, layers):
    """Distinct KV caches to rotate through so that one layer call never finds the previous
    call's KV in the 126 MB L2 (at least 4x L2 between reuses)."""
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    need = math.ceil(4 * l2 / max(kv_bytes_per_layer, 1))
    return int(max(1, min(layers, need)))


class StepState:
    """One workload's device inputs and the VerifyStep that runs it."""

    def __init__(self, cfg, device, seed):
        from speculative_decoding_verification_survival_b200 import VerifyStep

        self.cfg = cfg
        inp = build_step_inputs(cfg, device, seed=seed, layers=cfg.layers)
        kv_cache_bytes = inp.kv_caches[0].numel() * inp.kv_caches[0].element_size()
        self.copies = kv_copies_for(cfg, kv_cache_bytes, cfg.layers)
        if self.copies > 1:
            del inp
            inp = build_step_inputs(cfg, device, seed=seed, layers=cfg.layers,
                                    kv_copies=self.copies)
        self.inp = inp
        self.greedy = cfg.temperature <= 0
        self.step = VerifyStep(cfg.R, cfg.K, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, device=device)
        # the step is deterministic: schedule once to lay the target logits out per verify token
        self.step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
        torch.cuda.synchronize()
        self.L = self.step.verify_len.cpu().numpy()
        self.tflat = flatten_target(inp.target_block, self.L, cfg.T_cap)
        del inp.target_block
        torch.cuda.empty_cache()
        self.layers = [(inp.q[i], inp.k_new[i], inp.v_new[i]) for i in range(cfg.layers)]
        self.caches = [inp.kv_caches[i % self.copies] for i in range(cfg.layers)]
        self.attn_out = torch.empty_like(inp.q[0])
        self.dlog = None if self.greedy else inp.draft_logits

    def one_step(self, ev=None):
        inp, st = self.inp, self.step
        st.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
        st.plan(inp.kv_len)
        # the layer calls run back to back (each may start its prologue under the previous
        # one's tail); events bracket the whole run of them, not each call
        if ev is not None:
            ev[0].record()
        for (q, kn, vn), kv in zip(self.layers, self.caches):
            st.attention(q, kn, vn, kv, inp.block_table, inp.kv_len, self.attn_out)
        if ev is not None:
            ev[1].record()
        st.accept(self.tflat, self.dlog, inp.draft_tokens, inp.u_acc, inp.u_res,
                  self.cfg.temperature)


def run_dspark(args, cfg, rank, world, device, with_e2e=True):
    torch.cuda.set_device(device)
    S = StepState(cfg, device, seed=rank)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        S.one_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    launches_per_step = 2 + cfg.layers + 2
    # eager steps, for reference (every launch enqueued from the host)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_eager = min(args.steps, 5)
    e0.record(stream)
    for _ in range(n_eager):
        S.one_step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_eager = e0.elapsed_time(e1) / n_eager

    # the timed region: the K steps captured as one CUDA graph (every launch is sized by
    # capacities, so the steps need nothing from the host) and replayed once; events inside
    # the graph bracket each step's run of attention calls
    ev_attn = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
               for _ in range(args.steps)]

    def timed_steps():
        for s in range(args.steps):
            S.one_step(ev_attn[s])

    graph = S.step.capture(timed_steps, warmup=0)
    graph.replay()          # first replay uploads the graph; untimed
    torch.cuda.synchronize()

    def timed_replay():
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            t0.record(stream)
            graph.replay()
            t1.record(stream)
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        attn = [ev[0].elapsed_time(ev[1]) / cfg.layers for ev in ev_attn]
        return (t0.elapsed_time(t1), attn), clk.summary()

    # a run whose clock record shows a slowdown (or a leftover clock lock) is measured again
    (ms_total, attn_ms), clocks = measure_with_retry(
        timed_replay, lambda flag: agree_any(flag, device, world))
    del graph

    e2e = run_e2e(args, S, world, device) if with_e2e else None
    draft_ms = time_markov_draft(cfg, device) if cfg.dtype == "bf16" and cfg.V % 8 == 0 else None

    kv_len = S.inp.kv_len.cpu().numpy()
    acc = S.step.accepted_len.cpu().numpy()
    L = S.L
    res = dict(ms_total=ms_total, attn_ms=float(np.mean(attn_ms)), L=L, kv_len=kv_len, acc=acc,
               ms_eager=ms_eager, draft_ms=draft_ms,
               clocks=clocks, launches=launches_per_step * args.steps, e2e=e2e,
               attn_bytes=attn_bytes(kv_len, L, cfg),
               step_bytes=cfg.layers * attn_bytes(kv_len, L, cfg) + logits_bytes(L, cfg, S.greedy),
               step_bytes_strict=cfg.layers * attn_bytes(kv_len, L, cfg)
               + logits_bytes_strict(L, acc, cfg, S.greedy),
               kv_copies=S.copies)
    return S, res


def run_e2e(args, S, world, device):
    """The step through VerifyStep.run_from_host: every step copies its inputs from pinned host
    memory (on a copy stream, each call waiting only for its own inputs) and reads its results
    back; the results must equal the device-resident step's."""
    cfg, inp, step = S.cfg, S.inp, S.step
    stream = torch.cuda.current_stream()
    h = lambda t: t.detach().cpu().pin_memory() if t is not None else None
    host_in = dict(conf=h(inp.conf_ring), kv_len=h(inp.kv_len), t_ms=h(inp.t_ms),
                   q=h(inp.q), k_new=h(inp.k_new), v_new=h(inp.v_new), target_logits=h(S.tflat),
                   draft_logits=h(S.dlog), draft_tokens=h(inp.draft_tokens), u_acc=h(inp.u_acc),
                   u_res=h(inp.u_res))
    dev_in = {k: (torch.empty_like(v, device=device) if v is not None else None)
              for k, v in host_in.items()}
    names = ("verify_len", "accepted_len", "out_tokens", "n_out")
    expect = {k: getattr(step, k).cpu().numpy().copy() for k in names}  # the timed steps'
    host_out = {k: torch.empty(getattr(step, k).shape, dtype=getattr(step, k).dtype,
                               pin_memory=True) for k in names}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    attn_out = torch.empty_like(inp.q[0])
    copy_stream = torch.cuda.Stream(device=device)

    def one():
        step.run_from_host(host_in, dev_in, inp.round_idx, inp.block_table, S.caches, attn_out,
                           cfg.temperature, copy_stream, host_out)

    for _ in range(max(1, min(args.warmup, 3))):
        one()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    n = max(1, min(args.steps, 10))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    ok = all(np.array_equal(host_out[k].numpy(), expect[k]) for k in names)
    del host_in, dev_in
    return dict(ms=ms, h2d=h2d, d2h=d2h, ok=bool(ok))


# ---------------------------------------------------------------------------------------------
# The float64 oracle on the step's own inputs: parity of the benched step, and the CPU baseline.

def _host(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def request_pages(S, r):
    """Request r's cache pages (copy 0), its block-table row renumbered to them, and its
    cached length, on the host."""
    cfg, inp = S.cfg, S.inp
    n = int(inp.kv_len[r])
    npg = max(1, -(-n // cfg.page_size))
    pages = inp.block_table[r, :npg].long()
    local = _host(inp.kv_caches[0].index_select(0, pages.to(inp.kv_caches[0].device)))
    return local, np.arange(npg, dtype=np.int32)[None, :], n


def request_attn_inputs(S, r, qo, mk, layer=0):
    """Everything attn_ref_flat needs for request r alone (its tokens renumbered from 0)."""
    inp = S.inp
    local, table, n = request_pages(S, r)
    t0, t1 = int(qo[r]), int(qo[r + 1])
    markers = np.stack([np.zeros(t1 - t0, np.int32), mk[t0:t1, 1]], axis=1)
    return dict(q=_host(inp.q[layer, t0:t1]), k_new=_host(inp.k_new[layer, t0:t1]),
                v_new=_host(inp.v_new[layer, t0:t1]), kv_pages=local, block_table=table,
                kv_len=np.array([n]), markers=markers, q_offsets=np.array([0, t1 - t0]))


def split_by_kv_head(d, G):
    """The same request's attention as Hkv independent problems, one per KV head (its G query
    heads, its K/V rows): exactly the same arithmetic, in pieces a process pool can balance."""
    Hkv = d["k_new"].shape[1]
    return [dict(d, q=d["q"][:, g * G:(g + 1) * G], k_new=d["k_new"][:, g:g + 1],
                 v_new=d["v_new"][:, g:g + 1], kv_pages=d["kv_pages"][:, :, g:g + 1].copy())
            for g in range(Hkv)]


def _oracle_attn_task(args):
    """One request's attention in the oracle (every token, every query head); seconds taken."""
    from threadpoolctl import threadpool_limits
    import oracle
    d, scale, page = args
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle.attn_ref_flat(d["q"], d["k_new"], d["v_new"], d["kv_pages"], d["block_table"],
                             d["kv_len"], d["markers"], d["q_offsets"], scale, page)
        return time.perf_counter() - t0


def _oracle_accept_task(args):
    """A chunk of requests' acceptance in the oracle; (result, seconds taken)."""
    from threadpoolctl import threadpool_limits
    import oracle
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        res = oracle.accept_ref(*args)
        return res, time.perf_counter() - t0


def accept_chunk_args(S, r0, r1, qo):
    inp, cfg = S.inp, S.cfg
    a, b = int(qo[r0]), int(qo[r1])
    dl = (_host(inp.draft_logits[r0:r1]) if not S.greedy
          else np.zeros((r1 - r0, 1, 1), np.float32))
    return (_host(S.tflat[a:b]), dl, _host(inp.draft_tokens[r0:r1]), S.L[r0:r1],
            np.asarray(qo[r0:r1 + 1]) - a, _host(inp.u_acc[r0:r1]), _host(inp.u_res[r0:r1]),
            cfg.temperature)


def parity_check(S, attn_rows: int = 24):
    """The benched step against the oracle on the same input bits: the schedule (exact), every
    request's acceptance (exact except decisions the oracle flags within 1e-6 of a threshold,
    which are counted) and sampled attention rows of the last layer call (stated tolerance)."""
    import oracle
    from oracle.schedule import lagged_round

    cfg, inp, step = S.cfg, S.inp, S.step
    t_start = time.perf_counter()
    kv = _host(inp.kv_len).astype(np.int64)
    sref = oracle.schedule_ref(inp.conf_history[lagged_round(inp.round_idx)], kv,
                               _host(inp.t_ms), cfg.T_cap)
    T = int(step.T.item())
    sched_same = (np.array_equal(_host(step.verify_len), sref["verify_len"])
                  and np.array_equal(_host(step.q_offsets), sref["q_offsets"])
                  and np.array_equal(_host(step.markers)[:T], sref["markers"]))
    qo, mk = sref["q_offsets"], sref["markers"]
    got = {k: _host(getattr(step, k)) for k in ("accepted_len", "out_tokens", "n_out")}
    flagged = differ_flagged = differ_unflagged = 0
    chunk = 16
    for r0 in range(0, cfg.R, chunk):
        r1 = min(cfg.R, r0 + chunk)
        ref, _ = _oracle_accept_task(accept_chunk_args(S, r0, r1, qo))
        same = ((got["accepted_len"][r0:r1] == ref["accepted_len"])
                & np.all(got["out_tokens"][r0:r1] == ref["out_tokens"], axis=1)
                & (got["n_out"][r0:r1] == ref["n_out"]))
        flagged += int(ref["flagged"].sum())
        differ_flagged += int((~same & ref["flagged"]).sum())
        differ_unflagged += int((~same & ~ref["flagged"]).sum())
    # attention: sampled (token, head) rows of the last layer call, whose output the buffer holds
    layer = cfg.layers - 1
    rng = np.random.default_rng(7)
    toks = sorted(set(rng.integers(0, T, size=attn_rows).tolist()))
    out = S.attn_out
    errs = []
    scale = 1.0 / math.sqrt(cfg.D)
    for t in toks:
        r = int(mk[t, 0])
        d = request_attn_inputs(S, r, qo, mk, layer=layer)
        # the cache this layer call read
        if S.copies > 1:
            n = int(kv[r])
            npg = max(1, -(-n // cfg.page_size))
            pages = inp.block_table[r, :npg].long()
            d["kv_pages"] = _host(S.caches[layer].index_select(0, pages))
        h = int(rng.integers(0, cfg.Hq))
        ref = oracle.attn_ref_flat(d["q"], d["k_new"], d["v_new"], d["kv_pages"],
                                   d["block_table"], d["kv_len"], d["markers"], d["q_offsets"],
                                   scale, cfg.page_size, rows=[(t - int(qo[r]), h)])
        errs.append(np.abs(_host(out[t, h]).astype(np.float64) - ref[t - int(qo[r]), h]))
    errs = np.concatenate(errs)
    return dict(schedule="exact" if sched_same else ("flagged" if sref["flagged"] else "MISMATCH"),
                accept_requests=cfg.R, accept_flagged=flagged,
                accept_flagged_and_different=differ_flagged,
                accept_unflagged_mismatches=differ_unflagged,
                attention_rows=len(toks), attention_max_abs_err=float(errs.max()),
                attention_mean_abs_err=float(errs.mean()),
                seconds=time.perf_counter() - t_start)


def cpu_sample(cfg, kv, L, budget_units: float):
    """The bounded sample the CPU baseline times: whole requests in a fixed seeded order until
    their attention work (query rows x visible keys x D) reaches the budget, and as many
    requests' acceptance (up to 64).  Deterministic, so every leg times the same requests."""
    order = np.random.default_rng(0).permutation(cfg.R)
    units = (1 + L) * cfg.Hq * (kv + 1 + L) * cfg.D
    picked, tot = [], 0.0
    for r in order:
        picked.append(int(r))
        tot += float(units[r])
        if tot >= budget_units:
            break
    return picked, min(cfg.R, 64), float(units.sum()), float(sum(units[r] for r in picked))


# oracle attention work (query rows x visible keys x D) of the sample: about 20 s for one host
# thread (the oracle does ~1.1e8 such units per second and thread on the build host)
CPU_SAMPLE_UNITS = 2.0e9


def oracle_pool(n):
    """Worker processes for the oracle (spawned: a fork after CUDA initialisation can hang)."""
    ctx = mp.get_context("spawn")
    pool = ctx.Pool(n)
    pool.map(_noop, range(n))     # workers started and imported before anything is timed
    return pool


def _noop(_):
    return 0


def cpu_baseline(S, pool, n_workers, single_thread=True):
    """The float64 oracle timed on a bounded sample of the step and scaled to one whole step:
    the schedule of every request, the attention of the sampled requests (one layer call,
    scaled by attention work to every request and to `layers` calls), the acceptance of a
    prefix of requests (scaled to all).  Timed single-threaded and spread over `n_workers`
    processes of one thread each.  Returns the line's cpu_baseline object."""
    import oracle
    from oracle.schedule import lagged_round
    from threadpoolctl import threadpool_info, threadpool_limits

    cfg, inp = S.cfg, S.inp
    kv = _host(inp.kv_len).astype(np.int64)
    picked, n_acc, all_units, sample_units = cpu_sample(cfg, kv, S.L, CPU_SAMPLE_UNITS)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        s = oracle.schedule_ref(inp.conf_history[lagged_round(inp.round_idx)], kv,
                                _host(inp.t_ms), cfg.T_cap)
        t_sched = time.perf_counter() - t0
    qo, mk = s["q_offsets"], s["markers"]
    scale = 1.0 / math.sqrt(cfg.D)
    attn_tasks = [(part, scale, cfg.page_size) for r in picked
                  for part in split_by_kv_head(request_attn_inputs(S, r, qo, mk), cfg.G)]
    acc_tasks = [accept_chunk_args(S, r0, min(n_acc, r0 + 4), qo) for r0 in range(0, n_acc, 4)]

    def scaled(t_attn, t_acc):
        return t_sched + t_attn * (all_units / sample_units) * cfg.layers + t_acc * cfg.R / n_acc

    # one thread
    t_attn1 = t_acc1 = step1 = None
    if single_thread:
        t_attn1 = sum(_oracle_attn_task(a) for a in attn_tasks)
        t_acc1 = sum(_oracle_accept_task(a)[1] for a in acc_tasks)
        step1 = scaled(t_attn1, t_acc1)
    # all workers (wall time of the sample spread over the pool)
    t0 = time.perf_counter()
    pool.map(_oracle_attn_task, attn_tasks, chunksize=1)
    t_attn_n = time.perf_counter() - t0
    t0 = time.perf_counter()
    pool.map(_oracle_accept_task, acc_tasks, chunksize=1)
    t_acc_n = time.perf_counter() - t0
    stepn = scaled(t_attn_n, t_acc_n)
    tokens = float(S.L.sum())
    blas = [dict(api=i.get("internal_api"), threads=i.get("num_threads")) for i in threadpool_info()]
    sample = (f"oracle (float64 NumPy), one layer call's attention of {len(picked)} whole requests "
              f"(every token and head, one task per KV head; {sample_units / all_units:.4f} of the "
              f"call's work) scaled "
              f"to {cfg.R} requests x {cfg.layers} calls, acceptance of {n_acc} requests scaled "
              f"to {cfg.R}, schedule of all {cfg.R}; run on {n_workers} worker processes of one "
              f"thread each (single-thread figure beside it)")
    return dict(value=tokens / stepn, unit=UNIT, cores=n_workers, kind="oracle", sample=sample,
                est_step_s=stepn,
                single_thread=(dict(value=tokens / step1, est_step_s=step1) if single_thread
                               else None),
                sample_seconds=dict(attention=t_attn_n, accept=t_acc_n, schedule=t_sched,
                                    attention_1thread=t_attn1, accept_1thread=t_acc1),
                host_cores=len(os.sched_getaffinity(0)), blas_threads=blas)


def time_markov_draft(cfg, device, rounds: int = 10, rank: int = 64) -> float:
    """ms per round of the synthetic Markov-head draft step (the drafter's sequential part:
    K positions of block logits + a rank-64 previous-token transition, bf16 rounding and
    Gumbel-max sampling) for the workload's R, K, V; weights are random multiples of 1/16."""
    from speculative_decoding_verification_survival_b200 import dspark as d
    g = torch.Generator(device=device).manual_seed(0)
    R, K, V = cfg.R, cfg.K, cfg.V
    B = (torch.randn((R, K, V), generator=g, device=device) * 3).to(torch.bfloat16)
    E = (torch.randint(-16, 17, (V, rank), generator=g, device=device).float() / 16).to(torch.bfloat16)
    U = (torch.randint(-16, 17, (rank, V), generator=g, device=device).float() / 16).to(torch.bfloat16)
    x0 = torch.randint(0, V, (R,), generator=g, device=device, dtype=torch.int32)
    out = torch.empty_like(B)
    tok = torch.empty((R, K), dtype=torch.int32, device=device)
    ws = torch.empty(d.dspark_markov_draft_workspace_bytes(R, V), dtype=torch.uint8, device=device)
    tau = cfg.temperature
    for i in range(3):
        d.dspark_markov_draft(B, E, U, x0, tau, i, 0, out, tok, ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(rounds):
        d.dspark_markov_draft(B, E, U, x0, tau, i, 0, out, tok, ws)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / rounds
    del B, E, U, out
    return ms


def reduce_replicas(ms_step, attn_ms, e2e_ms, L_sum, acc_sum, R, world, device):
    """Combine independent replicas: times are the max over ranks (the job waits for the
    slowest), token and request counts are summed (every rank verifies its own batch)."""
    vec = torch.tensor([ms_step, attn_ms, e2e_ms, L_sum, acc_sum, R], dtype=torch.float64,
                       device=device)
    mx, sm = vec, vec
    if world > 1:
        mx = vec.clone()
        torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
        sm = vec.clone()
        torch.distributed.all_reduce(sm, op=torch.distributed.ReduceOp.SUM)
    return dict(ms_step=float(mx[0]), attn_ms=float(mx[1]), e2e_ms=float(mx[2]),
                L_tot=float(sm[3]), acc_tot=float(sm[4]), R_tot=float(sm[5]))


def bench_line(args, cfg, res, agg, world):
    peak, peak_kind = measured_peaks()
    ms_step, attn_ms, e2e_ms = agg["ms_step"], agg["attn_ms"], agg["e2e_ms"]
    L_tot, acc_tot, R_tot = agg["L_tot"], agg["acc_tot"], agg["R_tot"]
    achieved = res["attn_bytes"] / (attn_ms * 1e-3) / 1e9
    step_gbs = res["step_bytes"] / (ms_step * 1e-3) / 1e9
    line = dict(
        metric=METRIC, value=L_tot / (ms_step * 1e-3), unit=UNIT, n_gpus=world,
        steps=args.steps, warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
        scaling="weak", vs_baseline=None, dtype="bf16" if cfg.dtype == "bf16" else "f32",
        data="synthetic",
        config=dict(workload=cfg.name, R=cfg.R, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, V=cfg.V,
                    page_size=cfg.page_size, layers=cfg.layers, max_draft=cfg.K,
                    temperature=cfg.temperature, parallelism=f"replicas x{world}",
                    l2=f"inputs larger than L2: {res['attn_bytes'] / 1e9:.2f} GB of KV per "
                       f"layer call, {res['kv_copies']} distinct cache(s) rotated"),
        accepted_tokens_per_s=acc_tot / (ms_step * 1e-3),
        emitted_tokens_per_s=(acc_tot + R_tot) / (ms_step * 1e-3),
        mean_verify_len=L_tot / R_tot, mean_accepted=acc_tot / R_tot,
        step_hbm_gbs=step_gbs, step_frac_of_8tbs=step_gbs / 8000.0,
        step_frac_of_measured=step_gbs / peak,
        strict_lower_bound=dict(
            bytes_per_step=res["step_bytes_strict"],
            hbm_gbs=res["step_bytes_strict"] / (ms_step * 1e-3) / 1e9,
            frac_of_measured=res["step_bytes_strict"] / (ms_step * 1e-3) / 1e9 / peak,
            rows="logit rows only up to each request's first rejection"),
        roofline=dict(bound="hbm", kernel="dspark_verify_attn", achieved=achieved, peak=peak,
                      unit="GB/s", frac=achieved / peak, frac_of_8tbs=achieved / 8000.0,
                      traffic=measured_traffic(cfg.name, res["attn_bytes"]),
                      peak_source=peak_kind,
                      bytes_per_launch=res["attn_bytes"], ms_per_launch=attn_ms),
        gpu_launches=res["launches"] * world,
        launch=dict(timed="one CUDA graph of the K steps, replayed once",
                    ms_per_step_eager=res["ms_eager"]),
        draft_step=None if res["draft_ms"] is None else dict(
            ms_per_round=res["draft_ms"], share_of_verify_step=res["draft_ms"] / ms_step,
            model="Markov head: block logits (given) + rank-64 previous-token transition, "
                  "bf16 rounding, Gumbel-max; not part of the timed step"),
        clocks=res["clocks"])
    if res["e2e"] is not None:
        line["e2e"] = dict(value=L_tot / (e2e_ms * 1e-3), unit=UNIT,
                           h2d_bytes_per_step=res["e2e"]["h2d"],
                           d2h_bytes_per_step=res["e2e"]["d2h"],
                           ms_per_step=e2e_ms, results_match=res["e2e"]["ok"])
    return line


def run_reference(args, rank):
    """The reference arm: the oracle as it stands, on the host cores, one bounded sample of the
    workload per step (the sample the default run's cpu_baseline leg times)."""
    if rank != 0:
        return
    cfg = CONFIGS[args.workload].with_(layers=args.layers)
    device = "cuda" if torch.cuda.is_available() else "cpu"

    class _Inputs:       # the StepState fields the oracle legs read, without the CUDA library
        pass

    S = _Inputs()
    S.cfg = cfg
    S.inp = build_step_inputs(cfg.with_(layers=1), device, seed=0, layers=1)
    S.greedy = cfg.temperature <= 0
    import oracle
    from oracle.schedule import lagged_round
    s = oracle.schedule_ref(S.inp.conf_history[lagged_round(S.inp.round_idx)],
                            _host(S.inp.kv_len), _host(S.inp.t_ms), cfg.T_cap)
    S.L = s["verify_len"]
    S.tflat = flatten_target(S.inp.target_block, S.L, cfg.T_cap)
    n_workers = len(os.sched_getaffinity(0))
    pool = oracle_pool(n_workers)
    vals = []
    for _ in range(args.warmup + args.steps):   # each step: the sample on every host core
        vals.append(cpu_baseline(S, pool, n_workers, single_thread=False))
    timed = vals[args.warmup:]
    value = statistics.median(v["value"] for v in timed)
    ms = statistics.median(v["est_step_s"] for v in timed) * 1e3
    one = cpu_baseline(S, pool, n_workers, single_thread=True)   # once, for the record
    pool.close()
    cb = dict(timed[-1], value=value, single_thread=one["single_thread"])
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=cfg.name, R=cfg.R, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D,
                            V=cfg.V, layers=cfg.layers, max_draft=cfg.K,
                            temperature=cfg.temperature),
                cpu_baseline=cb,
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def report_row(line):
    p = line.get("parity", {})
    r = line["roofline"]
    return (f"| {line['config']['workload']} | {line['config']['R']} | "
            f"{line['mean_verify_len']:.2f} | {line['mean_accepted']:.2f} | "
            f"{line['value']:.0f} | {line['accepted_tokens_per_s']:.0f} | "
            f"{line['emitted_tokens_per_s']:.0f} | {line['ms_per_step']:.2f} | "
            f"{r['ms_per_launch'] * 1e3:.1f} | {r['achieved']:.0f} | {r['frac']:.3f} | "
            f"{r['frac_of_8tbs']:.3f} | {line['step_hbm_gbs']:.0f} | "
            f"{line['step_frac_of_measured']:.3f} | {line['step_frac_of_8tbs']:.3f} | "
            f"{p.get('schedule', '-')} | {p.get('accept_flagged', '-')} / "
            f"{p.get('accept_unflagged_mismatches', '-')} | "
            f"{(line.get('clocks') or {}).get('sm_mhz', '-')} |")


REPORT_HEADER = (
    "| workload | R | mean verify length | mean accepted | verified draft tok/s | accepted "
    "tok/s | emitted tok/s | step ms | attention µs/call | attention GB/s | of measured | "
    "of 8 TB/s | step GB/s | step of measured | step of 8 TB/s | schedule vs oracle | "
    "accept flagged / unflagged mismatches | SM MHz |\n" + "|---" * 18 + "|")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(CONFIGS))
    ap.add_argument("--layers", type=int, default=36)
    ap.add_argument("--requests", type=int, default=None,
                    help="the workload with this many requests instead (a smaller case of the "
                         "same distributions, e.g. for an ncu capture)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--report", action="store_true",
                    help="every workload in turn (fewer steps each), one JSON line per workload")
    ap.add_argument("--report-md", default=None, help="also write the report as a markdown table")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    pool, n_workers = None, len(os.sched_getaffinity(0))
    if rank == 0 and not args.no_cpu_baseline and not args.report:
        pool = oracle_pool(n_workers)

    workloads = REPORT_WORKLOADS if args.report else [args.workload]
    rows = []
    for name in workloads:
        cfg = CONFIGS[name].with_(layers=args.layers)
        if args.requests:
            cfg = cfg.with_(R=args.requests, name=f"{cfg.name}@{args.requests}req")
        S, res = run_dspark(args, cfg, rank, world, device, with_e2e=not args.report)
        agg = reduce_replicas(res["ms_total"] / args.steps, res["attn_ms"],
                              res["e2e"]["ms"] if res["e2e"] else 0.0,
                              int(res["L"].sum()), int(res["acc"].sum()), cfg.R, world, device)
        if rank == 0:
            line = bench_line(args, cfg, res, agg, world)
            if not args.no_parity:
                line["parity"] = parity_check(S)
            if pool is not None:
                line["cpu_baseline"] = cpu_baseline(S, pool, n_workers)
            print(json.dumps(line), flush=True)
            rows.append(line)
        del S
        torch.cuda.empty_cache()
    if pool is not None:
        pool.close()
    if rank == 0 and args.report_md:
        with open(args.report_md, "w") as fh:
            fh.write(REPORT_HEADER + "\n" + "\n".join(report_row(l) for l in rows) + "\n")
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
