"""CPU oracle for the DSpark verify step — TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 NumPy restatements of what one confidence-scheduled verify step computes.
Only the test suite, the smoke check and the benchmark's CPU-baseline leg may import this
package; the product path (the CUDA library and its Python binding) never does and shares no
code with it.

Sources (four news write-ups of the DSpark paper; they print no formulas or code):
  [P1] mooersco.com, "刚融完500亿创始人亲自下场写代码DeepSeek不卷参数专治AI“嘴慢”"
       sections "2. 置信度调度验证" and the engineering table (rows "GPU流水线停滞",
       "内核利用率暴跌").
  [P2] new-universe.cn, "DSpark 的 661% 提速，是真突破还是数字游戏？"
       sections 一 (verify-then-resample, exactness), 3.2 (confidence scheduling).
  [P3] qwbw.cn, "DeepSeek服务器不再卡顿！DSpark加速60% - 80%，推理成本降40%"
       sections "DSpark的神奇之处" (greedy scheduler), "成本与质量的考量" (exactness).
  [P4] aibuzzwire.news, "DeepSeek DSpark speculative decoding 85 percent faster LLM
       inference", section "置信度计划、负载感知验证" (survival probabilities, global
       throughput maximisation).

Pinned by tests/test_oracle_*.py against closed forms, brute force, library routines run as
such, invariants and a chi-square test of the output distribution.  Parity status of each
function is stated in its module header.
"""
from .schedule import (survival_ref, schedule_ref, schedule_bruteforce, flatten_ref,  # noqa: F401
                       lagged_round, CONF_LAG)
from .attention import attn_ref_flat, attn_ref_dense  # noqa: F401
from .accept import accept_ref  # noqa: F401
from .kv_commit import kv_commit_ref  # noqa: F401
from .calibration import calibrate_ref, fit_temperature_ref, outcomes_from_accept  # noqa: F401
from .draft import markov_draft_ref  # noqa: F401
