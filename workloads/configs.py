"""Synthetic verify-step workloads.

Five workloads, shaped like the ones the DSpark write-ups describe (max draft 5, GQA heads of
dimension 128, vocabularies of ~150k, long KV, a math/code/chat domain mix).  The pages print
no dataset items and none are reproduced here: every tensor is seeded synthetic data.

Readings taken where the workload statements leave a field open (each is listed in the
design notes):
  * N(mu, x) means x is the standard deviation.
  * Block positions k run 1..5; draft logits at position k = target + N(0, sigma_d * k).
  * Confidence noise sigma = 0.3 for every workload (only the tiny one states it).
  * "Mixed domains, a third each" assigns domain r % 3 to request r.
  * The tiny workload uses page size 8 so that pages are crossed within 8..40 tokens.
  * Workloads 3 and 5 use target logits N(0, 3) and page size 64; workload 4 uses
    a=2.5, b=0.4 and the 6 ms + 0.003 ms*max(0, T-512) step-time table.
  * Workload 5's "domain mix as in config 2" is read as workload 3's thirds (workload 2 has
    a single domain).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple


@dataclass(frozen=True)
class Domain:
    name: str
    a: float          # confidence logit intercept:  c_k = sigmoid(a - b*k + N(0, conf_sigma))
    b: float          # confidence logit slope per block position
    draft_noise: float  # draft logits = target + N(0, draft_noise * k)


MATH = Domain("math", 3.0, 0.3, 0.3)
CODE = Domain("code", 2.7, 0.35, 0.35)
CHAT = Domain("chat", 1.8, 0.5, 0.6)
THIRDS = (MATH, CODE, CHAT)


@dataclass(frozen=True)
class StepConfig:
    name: str
    R: int                      # requests in the verify batch
    Hq: int                     # query heads
    Hkv: int                    # KV heads (GQA group size G = Hq / Hkv)
    D: int                      # head dimension
    page_size: int              # KV cache page size (tokens)
    kv_dist: Tuple              # ("uniform", lo, hi) | ("lognormal", median, sigma, cap)
    V: int                      # vocabulary size
    target_std: float           # target logits ~ N(0, target_std)
    domains: Tuple[Domain, ...]
    t_base_ms: float            # step-time table t(T) = base + slope * max(0, T - knee)
    t_slope_ms: float
    t_knee: int
    dtype: str = "bf16"         # "bf16" | "f32": dtype of q/k/v, KV cache and logits
    K: int = 5                  # max draft length
    temperature: float = 1.0    # sampling temperature; <= 0 means greedy verification
    conf_sigma: float = 0.3
    forced_reject_frac: float = 0.0   # share of requests whose confidences are pinned low
    forced_reject_conf: float = 0.05
    layers: int = 36            # attention calls per verify step

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T_cap(self) -> int:
        return self.R * (self.K + 1)

    def with_(self, **kw) -> "StepConfig":
        return replace(self, **kw)


TINY = StepConfig(
    name="tiny", R=4, Hq=2, Hkv=1, D=16, page_size=8, kv_dist=("uniform", 8, 40), V=32,
    target_std=2.0, domains=(Domain("tiny", 2.0, 0.5, 0.5),),
    t_base_ms=1.0, t_slope_ms=0.01, t_knee=8, dtype="f32", layers=1)

QWEN3_4B = StepConfig(
    name="qwen3-4b-64req", R=64, Hq=32, Hkv=8, D=128, page_size=64,
    kv_dist=("uniform", 512, 4096), V=151936, target_std=3.0,
    domains=(Domain("uniform", 2.5, 0.4, 0.4),),
    t_base_ms=6.0, t_slope_ms=0.003, t_knee=512)

MIXED_256 = StepConfig(
    name="mixed-256req", R=256, Hq=40, Hkv=8, D=128, page_size=64,
    kv_dist=("uniform", 2048, 16384), V=151936, target_std=3.0, domains=THIRDS,
    t_base_ms=6.0, t_slope_ms=0.003, t_knee=512)

LONG_1024 = StepConfig(
    name="lognormal-1024req", R=1024, Hq=64, Hkv=8, D=128, page_size=64,
    kv_dist=("lognormal", 4096, 0.8, 32768), V=129280, target_std=4.0,
    domains=(Domain("uniform", 2.5, 0.4, 0.4),), temperature=0.7,
    t_base_ms=6.0, t_slope_ms=0.003, t_knee=512, forced_reject_frac=0.005)

SWEEP_LEVELS = (1, 8, 32, 128, 512, 1024, 2048)


def sweep_config(R: int) -> StepConfig:
    return StepConfig(
        name=f"sweep-{R}req", R=R, Hq=32, Hkv=8, D=128, page_size=64,
        kv_dist=("uniform", 1024, 8192), V=151936, target_std=3.0, domains=THIRDS,
        t_base_ms=5.0, t_slope_ms=0.004, t_knee=256)


# the same workload verified greedily (the workload statement asks for greedy and T=0.7 runs)
LONG_1024_GREEDY = LONG_1024.with_(name="lognormal-1024req-greedy", temperature=0.0)

CONFIGS = {
    "tiny": TINY,
    "qwen3-4b-64req": QWEN3_4B,
    "mixed-256req": MIXED_256,
    "lognormal-1024req": LONG_1024,
    "lognormal-1024req-greedy": LONG_1024_GREEDY,
}
for _R in SWEEP_LEVELS:
    CONFIGS[f"sweep-{_R}req"] = sweep_config(_R)
