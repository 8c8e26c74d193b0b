"""Verify rounds replayed as CUDA graphs, chained on the device.

"刚融完500亿…专治AI“嘴慢”", engineering table row "GPU流水线停滞": CUDA-graph replay needs the
next batch's size fixed in advance, and waiting for the current round's results to schedule the
next one leaves the GPU idle; the asynchronous scheduler therefore decides a round's verify
lengths from the confidences of two rounds earlier.  Here every launch is sized by capacity
(T_cap), so one captured graph serves every round whose scheduler reads the same confidence-ring
slot; a round is one replay:

    schedule (confidences of round i - 2) -> attention plan -> attention per layer -> accept
      -> KV commit (kept rows into the paged cache) -> kv_len <- kv_len_out

and the next round's replay reads the committed lengths from the same device buffer — nothing
returns to the host between rounds.  The caller (the engine) refills the round's input buffers
(queries, new K/V, logits, draft tokens, uniforms, the confidence-ring slot) before each replay.

With `overlap=True` the scheduler's decision for round i + 1 (survival scan, sort and greedy
prefix, which read only the lagged confidences) runs on a second stream while round i's
attention runs, into the other of two alternating sets of step buffers; round i + 1 then only
flattens its markers from the committed cache lengths before its attention plan.  The results
are the same as the serial chain's.
"""
from __future__ import annotations

import torch

from .step import VerifyStep

CONF_RING_LAG = 2


class RoundPipeline:
    def __init__(self, step: VerifyStep, conf_ring, t_ms, kv_len, block_table, q, k_new, v_new,
                 kv_caches, attn_out, target_logits, draft_logits, draft_tokens, u_acc, u_res,
                 temperature: float, overlap: bool = False):
        """q [layers][T_cap][Hq][D], k_new / v_new [layers][T_cap][Hkv][D] and kv_caches
        [layers][P][2][Hkv][page][D] are stacked per layer; every tensor is a fixed buffer the
        graphs capture by address."""
        self.step = step
        self.conf_ring, self.t_ms, self.kv_len, self.block_table = conf_ring, t_ms, kv_len, block_table
        self.q, self.k_new, self.v_new, self.kv_caches = q, k_new, v_new, kv_caches
        self.attn_out = attn_out
        self.target_logits, self.draft_logits = target_logits, draft_logits
        self.draft_tokens, self.u_acc, self.u_res = draft_tokens, u_acc, u_res
        self.temperature = temperature
        self.kv_len_out = torch.empty_like(kv_len)
        self.ring_depth = conf_ring.shape[0]
        self.overlap = overlap
        self.steps = [step]
        if overlap:   # a second set of step buffers: round i uses steps[i % 2]
            self.steps.append(VerifyStep(step.R, step.K, step.Hq, step.Hkv, step.D, step.V,
                                         device=step.q_offsets.device, T_cap=step.T_cap))
            self.side = torch.cuda.Stream(device=step.q_offsets.device)
        self._graphs = {}
        self._scheduled = None   # overlap: the round whose lengths are already decided

    def _slot(self, round_idx: int) -> int:
        return max(round_idx - CONF_RING_LAG, 0) % self.ring_depth

    def step_of(self, round_idx: int) -> VerifyStep:
        """The step buffers round `round_idx` runs in."""
        return self.steps[round_idx % len(self.steps)]

    def _body(self, st: VerifyStep) -> None:
        st.plan(self.kv_len)
        for layer in range(self.q.shape[0]):
            st.attention(self.q[layer], self.k_new[layer], self.v_new[layer],
                         self.kv_caches[layer], self.block_table, self.kv_len, self.attn_out[layer])
        st.accept(self.target_logits, self.draft_logits, self.draft_tokens, self.u_acc,
                  self.u_res, self.temperature)
        st.commit(self.k_new, self.v_new, self.kv_caches, self.block_table, self.kv_len,
                  self.kv_len_out)
        self.kv_len.copy_(self.kv_len_out)

    def enqueue(self, round_idx: int) -> None:
        """One round, eagerly on the current stream (what a replay executes; with overlap, the
        round's lengths must already be decided: use round())."""
        if not self.overlap:
            st = self.step
            st.schedule(self.conf_ring, round_idx, self.kv_len, self.t_ms)
            self._body(st)
            return
        st, nxt = self.step_of(round_idx), self.step_of(round_idx + 1)
        cur = torch.cuda.current_stream()
        # round i + 1's decision on the side stream, concurrent with this round's work
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            nxt.schedule_lengths(self.conf_ring, round_idx + 1, self.t_ms)
        st.flatten(self.kv_len)
        self._body(st)
        cur.wait_stream(self.side)

    def round(self, round_idx: int, graph: bool = True) -> None:
        """Run round `round_idx`: replay its graph (captured, without executing, on first use),
        or enqueue it eagerly with graph=False.  With overlap, a round whose lengths the
        previous round did not decide (the first one) gets them decided first."""
        if self.overlap:
            if self._scheduled != round_idx:
                self.step_of(round_idx).schedule_lengths(self.conf_ring, round_idx, self.t_ms)
            key = (round_idx % 2, self._slot(round_idx + 1))
            rep = round_idx
        else:
            key = self._slot(round_idx)
            # any round index whose lagged confidences sit in this slot
            rep = key + CONF_RING_LAG
        if graph:
            g = self._graphs.get(key)
            if g is None:
                g = self.step.capture(lambda: self.enqueue(rep), warmup=0)
                self._graphs[key] = g
            g.replay()
        else:
            self.enqueue(round_idx)
        self._scheduled = round_idx + 1
