"""Benchmark of one DSpark confidence-scheduled verify step on B200.

A step = dspark_schedule + dspark_verify_attn_plan + `layers` x dspark_verify_attn + dspark_accept
over one batch of seeded synthetic inputs already resident in HBM.  Metric: verified draft
tokens/s per verify step (sum of scheduled verify lengths / step time), plus accepted and
emitted tokens/s and the achieved HBM bandwidth of the step and of its dominant kernel.
The timed region is one replay of the K steps captured as a CUDA graph (the library sizes every
launch by capacity, so consecutive steps need no host involvement); the eager step time is
reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dspark|reference]
                    [--workload qwen3-4b-64req] [--layers 36]

Multi-GPU runs (torchrun, one process per GPU) are independent replicas: each rank verifies its
own request batch (seed = rank) with no data-path collective; the step time is the max over
ranks and `value` sums every rank's tokens.  `--impl reference` times the float64 CPU oracle
on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
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

from workloads.configs import CONFIGS  # noqa: E402
from workloads.generate import build_step_inputs, flatten_target  # noqa: E402

METRIC = "verified draft tokens/s per verify step (1 B200); achieved HBM GB/s vs peak"
UNIT = "tokens/s"


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
        sm, mx, reasons = [], [], set()
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
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch, from an ncu
# capture of the bench's own command (the summary under profiles/ gives the command), keyed by the
# SHA-1 of the kernel sources the capture ran; any change to those sources voids the figure.
NCU_TRAFFIC = {
    # profiles/attn_tc_kernel_qwen3-4b-64req_full.md: 626.618624 MB read + 4.616192 MB written
    "qwen3-4b-64req": ("b7667a45921c3d9cfd3c89a9121bfc2c701ef656", 631234816),
}


def kernel_source_hash():
    import hashlib
    d = os.path.join(ROOT, "speculative_decoding_verification_survival_b200", "csrc")
    h = hashlib.sha1()
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(d, name), "rb") as fh:
                h.update(name.encode() + b"\0" + fh.read())
    return h.hexdigest()


def measured_traffic(workload):
    rec = NCU_TRAFFIC.get(workload)
    if rec is None or rec[0] != kernel_source_hash():
        return None
    return rec[1]


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


def run_dspark(args, rank, world, device):
    from speculative_decoding_verification_survival_b200 import VerifyStep

    cfg = CONFIGS[args.workload].with_(layers=args.layers)
    torch.cuda.set_device(device)
    inp = build_step_inputs(cfg, device, seed=rank, layers=cfg.layers)
    kv_cache_bytes = inp.kv_caches[0].numel() * inp.kv_caches[0].element_size()
    copies = kv_copies_for(cfg, kv_cache_bytes, cfg.layers)
    if copies > 1:
        del inp
        inp = build_step_inputs(cfg, device, seed=rank, layers=cfg.layers, kv_copies=copies)
    greedy = cfg.temperature <= 0
    step = VerifyStep(cfg.R, cfg.K, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, device=device)
    stream = torch.cuda.current_stream()

    # the step is deterministic: schedule once to lay the target logits out per verify token
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    torch.cuda.synchronize()
    L = step.verify_len.cpu().numpy()
    tflat = flatten_target(inp.target_block, L, cfg.T_cap)
    del inp.target_block
    torch.cuda.empty_cache()
    layers = [(inp.q[i], inp.k_new[i], inp.v_new[i]) for i in range(cfg.layers)]
    caches = [inp.kv_caches[i % copies] for i in range(cfg.layers)]
    attn_out = torch.empty_like(inp.q[0])
    dlog = None if greedy else inp.draft_logits

    def one_step(ev=None):
        step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
        step.plan(inp.kv_len)
        # the layer calls run back to back (each may start its prologue under the previous
        # one's tail); events bracket the whole run of them, not each call
        if ev is not None:
            ev[0].record()
        for (q, kn, vn), kv in zip(layers, caches):
            step.attention(q, kn, vn, kv, inp.block_table, inp.kv_len, attn_out)
        if ev is not None:
            ev[1].record()
        step.accept(tflat, dlog, inp.draft_tokens, inp.u_acc, inp.u_res, cfg.temperature)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    launches_per_step = 2 + cfg.layers + 2
    # eager steps, for reference (every launch enqueued from the host)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_eager = min(args.steps, 10)
    e0.record(stream)
    for _ in range(n_eager):
        one_step()
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
            one_step(ev_attn[s])

    graph = step.capture(timed_steps, warmup=0)
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

    # end to end through the public step API with host buffers (pinned), copies inside
    e2e = run_e2e(args, cfg, inp, step, layers, caches, tflat, dlog, L, world, device)
    draft_ms = time_markov_draft(cfg, device) if cfg.dtype == "bf16" and cfg.V % 8 == 0 else None

    kv_len = inp.kv_len.cpu().numpy()
    acc = step.accepted_len.cpu().numpy()
    res = dict(ms_total=ms_total, attn_ms=float(np.mean(attn_ms)), L=L, kv_len=kv_len, acc=acc,
               ms_eager=ms_eager, draft_ms=draft_ms,
               clocks=clocks, launches=launches_per_step * args.steps, e2e=e2e,
               attn_bytes=attn_bytes(kv_len, L, cfg),
               step_bytes=cfg.layers * attn_bytes(kv_len, L, cfg) + logits_bytes(L, cfg, greedy),
               step_bytes_strict=cfg.layers * attn_bytes(kv_len, L, cfg)
               + logits_bytes_strict(L, acc, cfg, greedy),
               kv_copies=copies)
    return cfg, res


def run_e2e(args, cfg, inp, step, layers, caches, tflat, dlog, L, world, device):
    """The step through VerifyStep.run_from_host: every step copies its inputs from pinned host
    memory (on a copy stream, each call waiting only for its own inputs) and reads its results
    back."""
    stream = torch.cuda.current_stream()
    h = lambda t: t.detach().cpu().pin_memory() if t is not None else None
    host_in = dict(conf=h(inp.conf_ring), kv_len=h(inp.kv_len), t_ms=h(inp.t_ms),
                   q=h(inp.q), k_new=h(inp.k_new), v_new=h(inp.v_new), target_logits=h(tflat),
                   draft_logits=h(dlog), draft_tokens=h(inp.draft_tokens), u_acc=h(inp.u_acc),
                   u_res=h(inp.u_res))
    dev_in = {k: (torch.empty_like(v, device=device) if v is not None else None)
              for k, v in host_in.items()}
    host_out = {k: torch.empty(getattr(step, k).shape, dtype=getattr(step, k).dtype,
                               pin_memory=True)
                for k in ("verify_len", "accepted_len", "out_tokens", "n_out")}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    attn_out = torch.empty_like(inp.q[0])
    copy_stream = torch.cuda.Stream(device=device)

    def one():
        step.run_from_host(host_in, dev_in, inp.round_idx, inp.block_table, caches, attn_out,
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
    ok = np.array_equal(host_out["verify_len"].numpy(), L)
    return dict(ms=ms, h2d=h2d, d2h=d2h, ok=bool(ok))


def cpu_baseline(cfg, max_seconds: float = 20.0):
    """The float64 oracle, single-threaded, timed on a bounded sample of the workload and
    scaled to one full step; returns (verified draft tokens/s, description, cores)."""
    from threadpoolctl import threadpool_limits

    import oracle
    from oracle.schedule import lagged_round

    with threadpool_limits(limits=1):
        inp = build_step_inputs(cfg.with_(layers=1), "cpu", seed=0, layers=1)
        conf = inp.conf_history[lagged_round(inp.round_idx)]
        kv = inp.kv_len.numpy()
        t0 = time.perf_counter()
        s = oracle.schedule_ref(conf, kv, inp.t_ms.numpy(), cfg.T_cap)
        t_sched = time.perf_counter() - t0
        L, qo, mk = s["verify_len"], s["q_offsets"], s["markers"]
        # attention: whole requests (every token, every head) until the time budget is used
        order = np.random.default_rng(0).permutation(cfg.R)
        t_attn, done_kv, tot_kv = 0.0, 0, int((kv + 1 + L).sum())
        kvp = inp.kv_caches[0].float().numpy() if cfg.dtype == "bf16" else inp.kv_caches[0].numpy()
        q = inp.q[0].float().numpy()
        kn, vn = inp.k_new[0].float().numpy(), inp.v_new[0].float().numpy()
        bt = inp.block_table.numpy()
        nreq = 0
        for r in order:
            rows = [(t, h) for t in range(qo[r], qo[r + 1]) for h in range(cfg.Hq)]
            t0 = time.perf_counter()
            oracle.attn_ref_flat(q, kn, vn, kvp, bt, kv, mk, qo, 1.0 / math.sqrt(cfg.D),
                                 cfg.page_size, rows=rows)
            t_attn += time.perf_counter() - t0
            done_kv += int(kv[r] + 1 + L[r])
            nreq += 1
            if t_attn > max_seconds / 2:
                break
        t_attn_step = t_attn * tot_kv / done_kv * cfg.layers
        # acceptance: a prefix of requests
        tflat = flatten_target(inp.target_block, L, cfg.T_cap)
        t0 = time.perf_counter()
        nacc = 0
        for r0 in range(0, cfg.R, 4):
            r1 = min(cfg.R, r0 + 4)
            a, b = int(qo[r0]), int(qo[r1])
            oracle.accept_ref(tflat[a:b].float().numpy(), inp.draft_logits[r0:r1].float().numpy(),
                              inp.draft_tokens[r0:r1].numpy(), L[r0:r1], qo[r0:r1 + 1] - a,
                              inp.u_acc[r0:r1].numpy(), inp.u_res[r0:r1].numpy(), cfg.temperature)
            nacc = r1
            if time.perf_counter() - t0 > max_seconds / 2:
                break
        t_acc_step = (time.perf_counter() - t0) * cfg.R / nacc
    step_s = t_sched + t_attn_step + t_acc_step
    desc = (f"oracle, 1 thread: schedule of all {cfg.R} requests; attention of {nreq} whole "
            f"requests (all tokens and heads) scaled by KV rows to {cfg.R} requests x "
            f"{cfg.layers} layers; acceptance of {nacc} requests scaled to {cfg.R}")
    return float(L.sum()) / step_s, desc, 1, step_s


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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default="qwen3-4b-64req", choices=sorted(CONFIGS))
    ap.add_argument("--layers", type=int, default=36)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        cfg = CONFIGS[args.workload].with_(layers=args.layers)
        vals = []
        for _ in range(args.warmup + args.steps):
            v, desc, cores, step_s = cpu_baseline(cfg, max_seconds=6.0)
            vals.append((v, step_s))
        timed = vals[args.warmup:]
        value = statistics.median(v for v, _ in timed)
        ms = statistics.median(s for _, s in timed) * 1e3
        line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak",
                    vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                    config=dict(workload=cfg.name, R=cfg.R, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D,
                                V=cfg.V, layers=cfg.layers, max_draft=cfg.K),
                    cpu_baseline=dict(value=value, unit=UNIT, cores=cores, kind="oracle",
                                      sample=desc),
                    e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg, res = run_dspark(args, rank, world, device)

    R = cfg.R
    agg = reduce_replicas(res["ms_total"] / args.steps, res["attn_ms"], res["e2e"]["ms"],
                          int(res["L"].sum()), int(res["acc"].sum()), R, world, device)
    ms_step, attn_ms, e2e_ms = agg["ms_step"], agg["attn_ms"], agg["e2e_ms"]
    L_tot, acc_tot, R_tot = agg["L_tot"], agg["acc_tot"], agg["R_tot"]

    if rank == 0:
        peak, peak_kind = measured_peaks()
        achieved = res["attn_bytes"] / (attn_ms * 1e-3) / 1e9
        step_gbs = res["step_bytes"] / (ms_step * 1e-3) / 1e9
        line = dict(
            metric=METRIC, value=L_tot / (ms_step * 1e-3), unit=UNIT, n_gpus=world,
            steps=args.steps, warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
            scaling="weak", vs_baseline=None, dtype="bf16" if cfg.dtype == "bf16" else "f32",
            data="synthetic",
            config=dict(workload=cfg.name, R=R, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, V=cfg.V,
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
                          unit="GB/s", frac=achieved / peak,
                          traffic=measured_traffic(cfg.name),
                          peak_source=peak_kind,
                          bytes_per_launch=res["attn_bytes"], ms_per_launch=attn_ms),
            e2e=dict(value=L_tot / (e2e_ms * 1e-3), unit=UNIT,
                     h2d_bytes_per_step=res["e2e"]["h2d"], d2h_bytes_per_step=res["e2e"]["d2h"],
                     ms_per_step=e2e_ms, results_match=res["e2e"]["ok"]),
            gpu_launches=res["launches"] * world,
            launch=dict(timed="one CUDA graph of the K steps, replayed once",
                        ms_per_step_eager=res["ms_eager"]),
            draft_step=None if res["draft_ms"] is None else dict(
                ms_per_round=res["draft_ms"], share_of_verify_step=res["draft_ms"] / ms_step,
                model="Markov head: block logits (given) + rank-64 previous-token transition, "
                      "bf16 rounding, Gumbel-max; not part of the timed step"),
            clocks=res["clocks"])
        if not args.no_cpu_baseline:
            v, desc, cores, step_s = cpu_baseline(cfg)
            line["cpu_baseline"] = dict(value=v, unit=UNIT, cores=cores, kind="oracle",
                                        sample=desc, est_step_s=step_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
