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
"""
from __future__ import annotations

import torch

from .step import VerifyStep

CONF_RING_LAG = 2


class RoundPipeline:
    def __init__(self, step: VerifyStep, conf_ring, t_ms, kv_len, block_table, q, k_new, v_new,
                 kv_caches, attn_out, target_logits, draft_logits, draft_tokens, u_acc, u_res,
                 temperature: float):
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
        self._graphs = {}

    def _slot(self, round_idx: int) -> int:
        return max(round_idx - CONF_RING_LAG, 0) % self.ring_depth

    def enqueue(self, round_idx: int) -> None:
        """One round, eagerly on the current stream (what a replay executes)."""
        st = self.step
        st.schedule(self.conf_ring, round_idx, self.kv_len, self.t_ms)
        st.plan(self.kv_len)
        for layer in range(self.q.shape[0]):
            st.attention(self.q[layer], self.k_new[layer], self.v_new[layer],
                         self.kv_caches[layer], self.block_table, self.kv_len, self.attn_out[layer])
        st.accept(self.target_logits, self.draft_logits, self.draft_tokens, self.u_acc,
                  self.u_res, self.temperature)
        st.commit(self.k_new, self.v_new, self.kv_caches, self.block_table, self.kv_len,
                  self.kv_len_out)
        self.kv_len.copy_(self.kv_len_out)

    def round(self, round_idx: int) -> None:
        """Replay the graph of this round's confidence-ring slot (captured, without executing,
        on first use)."""
        slot = self._slot(round_idx)
        g = self._graphs.get(slot)
        if g is None:
            # any round index whose lagged confidences sit in this slot
            g = self.step.capture(lambda: self.enqueue(slot + CONF_RING_LAG), warmup=0)
            self._graphs[slot] = g
        g.replay()
