"""Seeded synthetic inputs for one verify step.

Everything here is input synthesis: KV lengths, a paged KV cache, per-layer queries, target and
draft logits, the drafted tokens, confidence histories, the engine's step-time table and the
acceptance uniforms.  None of the verification arithmetic (survival scan, scheduling,
attention, acceptance) lives here; both the CUDA path and the CPU oracle receive these arrays.

Small host-side arrays come from numpy's default_rng(seed); bulk tensors come from a seeded
torch.Generator on the requested device, so that multi-GB workloads are generated in HBM.
The oracle always reads back the exact bits the GPU received.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from .configs import StepConfig
from .philox import step_uniforms

CONF_RING = 3  # confidence history slots: the scheduler reads the round two steps back


def torch_dtype(cfg: StepConfig) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[cfg.dtype]


def kv_lengths(cfg: StepConfig, rng: np.random.Generator) -> np.ndarray:
    kind = cfg.kv_dist[0]
    if kind == "uniform":
        lo, hi = cfg.kv_dist[1], cfg.kv_dist[2]
        n = rng.integers(lo, hi + 1, size=cfg.R)
    elif kind == "lognormal":
        median, sigma, cap = cfg.kv_dist[1:4]
        n = np.exp(math.log(median) + sigma * rng.standard_normal(cfg.R))
        n = np.clip(np.rint(n), 1, cap)
    else:
        raise ValueError(f"unknown KV length distribution {kind!r}")
    return n.astype(np.int32)


def domain_of(cfg: StepConfig) -> np.ndarray:
    """Domain index per request: request r belongs to domain r % len(domains)."""
    return np.arange(cfg.R) % len(cfg.domains)


def confidences(cfg: StepConfig, rng: np.random.Generator, rounds: int) -> np.ndarray:
    """Confidence-head outputs c[round][r][k] = sigmoid(a - b*k + N(0, sigma)), k = 1..K.

    Requests chosen for forced rejection get c = forced_reject_conf at every position.
    """
    dom = domain_of(cfg)
    a = np.array([cfg.domains[d].a for d in dom])[:, None]
    b = np.array([cfg.domains[d].b for d in dom])[:, None]
    k = np.arange(1, cfg.K + 1, dtype=np.float64)[None, :]
    out = np.empty((rounds, cfg.R, cfg.K), dtype=np.float32)
    forced = forced_reject_mask(cfg)
    for i in range(rounds):
        logit = a - b * k + cfg.conf_sigma * rng.standard_normal((cfg.R, cfg.K))
        c = 1.0 / (1.0 + np.exp(-logit))
        c[forced] = cfg.forced_reject_conf
        out[i] = c.astype(np.float32)
    return out


def forced_reject_mask(cfg: StepConfig) -> np.ndarray:
    n = int(round(cfg.forced_reject_frac * cfg.R))
    mask = np.zeros(cfg.R, dtype=bool)
    if n > 0:
        # spread evenly through the batch so every domain / length band is touched
        mask[np.linspace(0, cfg.R - 1, n).round().astype(int)] = True
    return mask


def conf_ring(history: np.ndarray, round_idx: int) -> np.ndarray:
    """Pack the confidence history of rounds 0..round_idx into a CONF_RING-slot ring.

    Slot (i % CONF_RING) holds round i for the last CONF_RING rounds up to round_idx.
    """
    ring = np.zeros((CONF_RING,) + history.shape[1:], dtype=np.float32)
    for i in range(max(0, round_idx - CONF_RING + 1), round_idx + 1):
        ring[i % CONF_RING] = history[i]
    return ring


def step_time_table(cfg: StepConfig, T_cap: Optional[int] = None) -> np.ndarray:
    """Engine step time t_ms[T] for T = 0..T_cap verify tokens (the measured throughput curve)."""
    T_cap = cfg.T_cap if T_cap is None else T_cap
    T = np.arange(T_cap + 1, dtype=np.float64)
    return cfg.t_base_ms + cfg.t_slope_ms * np.maximum(0.0, T - cfg.t_knee)


def page_table(kv_len: np.ndarray, page_size: int, rng: np.random.Generator, reserve: int = 0):
    """Random physical placement of each request's KV pages, with room for `reserve` more
    tokens per request (the positions a verify round may append).

    Returns (block_table int32 [R][max_pages] padded with -1, num_pages).
    """
    pages_per = (kv_len.astype(np.int64) + reserve + page_size - 1) // page_size
    num_pages = int(pages_per.sum())
    max_pages = max(1, int(pages_per.max()) if len(pages_per) else 1)
    perm = rng.permutation(num_pages).astype(np.int32)
    table = np.full((len(kv_len), max_pages), -1, dtype=np.int32)
    off = 0
    for r, p in enumerate(pages_per):
        table[r, :p] = perm[off:off + p]
        off += p
    return table, max(num_pages, 1)


@dataclass
class StepInputs:
    cfg: StepConfig
    round_idx: int
    kv_len: torch.Tensor          # int32 [R]
    block_table: torch.Tensor     # int32 [R][max_pages]
    kv_caches: list               # kv_copies x dtype [num_pages][2][Hkv][page][D]
    q: torch.Tensor               # dtype [layers][T_cap][Hq][D]
    k_new: torch.Tensor           # dtype [layers][T_cap][Hkv][D]
    v_new: torch.Tensor           # dtype [layers][T_cap][Hkv][D]
    target_block: torch.Tensor    # dtype [R][K+1][V]: target logits for block positions 1..K+1
    draft_logits: torch.Tensor    # dtype [R][K][V]: draft logits for block positions 1..K
    draft_tokens: torch.Tensor    # int32 [R][K]
    conf_history: np.ndarray      # float32 [rounds][R][K]
    conf_ring: torch.Tensor       # float32 [CONF_RING][R][K]
    t_ms: torch.Tensor            # float64 [T_cap+1]
    u_acc: torch.Tensor           # float32 [R][K]
    u_res: torch.Tensor           # float32 [R][K+1]

    @property
    def num_pages(self) -> int:
        return self.kv_caches[0].shape[0]


def _normal(shape, std, gen, device, dtype):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def sample_draft_tokens(draft_logits: torch.Tensor, temperature: float,
                        gen: torch.Generator, chunk: int = 64) -> torch.Tensor:
    """Draft tokens x_k ~ softmax(draft_logits[k] / temperature) by the Gumbel-max trick
    (argmax of logits/temperature + Gumbel noise), or argmax when temperature <= 0."""
    R, K, V = draft_logits.shape
    out = torch.empty((R, K), dtype=torch.int32, device=draft_logits.device)
    for r0 in range(0, R, chunk):
        z = draft_logits[r0:r0 + chunk].float()
        if temperature > 0:
            u = torch.rand(z.shape, generator=gen, device=z.device, dtype=torch.float32)
            z = z / temperature - torch.log(-torch.log(u))
        out[r0:r0 + chunk] = torch.argmax(z, dim=-1).to(torch.int32)
    return out


def build_step_inputs(cfg: StepConfig, device="cpu", seed: int = 0, layers: Optional[int] = None,
                      rounds: int = 4, kv_copies: int = 1,
                      reserve_tokens: Optional[int] = None) -> StepInputs:
    """All inputs of verify round `rounds - 1` of workload `cfg`; the block table has room for
    `reserve_tokens` (default K + 1) appended tokens per request."""
    device = torch.device(device)
    layers = cfg.layers if layers is None else layers
    rng = np.random.default_rng(seed)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = torch_dtype(cfg)
    R, K, V = cfg.R, cfg.K, cfg.V

    kv_len = kv_lengths(cfg, rng)
    reserve = cfg.K + 1 if reserve_tokens is None else reserve_tokens
    table, num_pages = page_table(kv_len, cfg.page_size, rng, reserve=reserve)
    history = confidences(cfg, rng, rounds)
    round_idx = rounds - 1
    ring = conf_ring(history, round_idx)
    u_acc, u_res = step_uniforms(round_idx, R, K, seed)

    caches = [_normal((num_pages, 2, cfg.Hkv, cfg.page_size, cfg.D), 1.0, gen, device, dt)
              for _ in range(kv_copies)]
    q = _normal((layers, cfg.T_cap, cfg.Hq, cfg.D), 1.0, gen, device, dt)
    k_new = _normal((layers, cfg.T_cap, cfg.Hkv, cfg.D), 1.0, gen, device, dt)
    v_new = _normal((layers, cfg.T_cap, cfg.Hkv, cfg.D), 1.0, gen, device, dt)

    target_block = torch.empty((R, K + 1, V), dtype=dt, device=device)
    draft_logits = torch.empty((R, K, V), dtype=dt, device=device)
    dom = domain_of(cfg)
    sig = torch.tensor([cfg.domains[d].draft_noise for d in dom], dtype=torch.float32,
                       device=device)
    kpos = torch.arange(1, K + 1, dtype=torch.float32, device=device)
    chunk = max(1, (1 << 28) // (4 * (2 * K + 1) * V))
    for r0 in range(0, R, chunk):
        r1 = min(R, r0 + chunk)
        tb = torch.randn((r1 - r0, K + 1, V), generator=gen, device=device) * cfg.target_std
        noise = torch.randn((r1 - r0, K, V), generator=gen, device=device)
        scale = (sig[r0:r1, None] * kpos[None, :])[..., None]
        target_block[r0:r1] = tb.to(dt)
        draft_logits[r0:r1] = (tb[:, :K] + noise * scale).to(dt)
    draft_tokens = sample_draft_tokens(draft_logits, cfg.temperature, gen)

    as_dev = lambda a, dtype: torch.as_tensor(a, dtype=dtype).to(device)
    return StepInputs(
        cfg=cfg, round_idx=round_idx,
        kv_len=as_dev(kv_len, torch.int32), block_table=as_dev(table, torch.int32),
        kv_caches=caches, q=q, k_new=k_new, v_new=v_new,
        target_block=target_block, draft_logits=draft_logits, draft_tokens=draft_tokens,
        conf_history=history, conf_ring=as_dev(ring, torch.float32),
        t_ms=as_dev(step_time_table(cfg), torch.float64),
        u_acc=as_dev(u_acc, torch.float32), u_res=as_dev(u_res, torch.float32))


def flatten_target(target_block: torch.Tensor, verify_len, T_cap: int) -> torch.Tensor:
    """Target logits laid out as the target model emits them: one row per verify token.

    Request r's Q_r = 1 + verify_len[r] rows are contiguous and in block order; rows beyond the
    scheduled total are zero.  Pure data movement (a gather).
    """
    R, K1, V = target_block.shape
    L = torch.as_tensor(verify_len, dtype=torch.int64).cpu()
    out = torch.zeros((T_cap, V), dtype=target_block.dtype, device=target_block.device)
    t = 0
    for r in range(R):
        n = int(L[r]) + 1
        out[t:t + n] = target_block[r, :n]
        t += n
    return out
