"""One confidence-scheduled verify step on one GPU, composed from the libdspark entry points.

    schedule (lagged confidences -> verify lengths, offsets, markers)
      -> attention plan (work partition of the step, reused by every layer)
      -> one flattened verify-attention call per layer
      -> accept (acceptance test, longest prefix, correction / bonus token)

VerifyStep owns the step's device outputs and workspaces (allocated once through torch) and
issues the calls in order on the current stream.  It does no arithmetic of its own.
"""
from __future__ import annotations

import math

import torch

from . import dspark as _d


class VerifyStep:
    def __init__(self, R: int, K: int, Hq: int, Hkv: int, D: int, V: int, device="cuda",
                 T_cap: int | None = None):
        self.R, self.K, self.Hq, self.Hkv, self.D, self.V = R, K, Hq, Hkv, D, V
        self.T_cap = R * (K + 1) if T_cap is None else T_cap
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.verify_len = torch.zeros(R, **i32)
        self.q_offsets = torch.zeros(R + 1, **i32)
        self.markers = torch.zeros(self.T_cap, 2, **i32)
        self.T = torch.zeros(1, **i32)
        self.objective = torch.zeros(1, dtype=torch.float64, device=dev)
        self.accepted_len = torch.zeros(R, **i32)
        self.out_tokens = torch.zeros(R, K + 1, **i32)
        self.n_out = torch.zeros(R, **i32)
        nbytes = _d.dspark_verify_attn_workspace_bytes(R, Hq, Hkv, D, K)
        self.attn_ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
        nbytes = _d.dspark_accept_workspace_bytes(R, K, self.T_cap)
        self.accept_ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
        self.scale = 1.0 / math.sqrt(D)

    def schedule(self, conf_ring, round_idx, kv_len, t_ms, stream=None):
        _d.dspark_schedule(conf_ring, round_idx, kv_len, t_ms, self.T_cap, self.verify_len,
                           self.q_offsets, self.markers, self.T, self.objective, stream)

    def schedule_lengths(self, conf_ring, round_idx, t_ms, stream=None):
        """The schedule's decision alone (verify lengths, offsets, T, objective): it reads only
        the lagged confidences and the step-time table, so it may run before the previous
        round has committed its cache lengths; flatten() then writes the markers."""
        _d.dspark_schedule(conf_ring, round_idx, None, t_ms, self.T_cap, self.verify_len,
                           self.q_offsets, None, self.T, self.objective, stream)

    def flatten(self, kv_len, stream=None):
        """Markers of the scheduled lengths at the current cache lengths."""
        _d.dspark_flatten_markers(kv_len, self.q_offsets, self.K, self.markers, stream)

    def plan(self, kv_len, stream=None):
        _d.dspark_verify_attn_plan(kv_len, self.q_offsets, self.markers, self.R, self.Hq,
                                   self.Hkv, self.D, self.K, self.attn_ws, stream)

    def attention(self, q, k_new, v_new, kv_pages, block_table, kv_len, out, stream=None):
        _d.dspark_verify_attn(q, k_new, v_new, kv_pages, block_table, kv_len, self.markers,
                              self.q_offsets, self.K, self.scale, out, self.attn_ws, stream)

    def accept(self, target_logits, draft_logits, draft_tokens, u_acc, u_res, temperature,
               stream=None):
        _d.dspark_accept(target_logits, draft_logits, draft_tokens, self.verify_len,
                         self.q_offsets, u_acc, u_res, temperature, self.accepted_len,
                         self.out_tokens, self.n_out, self.accept_ws, stream)

    def commit(self, k_new, v_new, kv_pages, block_table, kv_len, kv_len_out, stream=None):
        """Append each request's kept verify rows (token 0 and its accepted drafts) to its paged
        cache for every layer; kv_len_out = kv_len + accepted + 1."""
        _d.dspark_kv_commit(k_new, v_new, kv_pages, block_table, kv_len, self.q_offsets,
                            self.accepted_len, self.K, kv_len_out, stream)

    INPUT_KEYS = ("conf", "kv_len", "t_ms", "q", "k_new", "v_new", "target_logits",
                  "draft_logits", "draft_tokens", "u_acc", "u_res")

    def run_from_host(self, host: dict, dev: dict, round_idx: int, block_table,
                      kv_pages_per_layer, attn_out, temperature: float, copy_stream,
                      host_out: dict | None = None) -> int:
        """One step whose inputs arrive from (pinned) host memory.

        `host` and `dev` map INPUT_KEYS to host tensors and same-shaped device buffers (q,
        k_new, v_new stacked per layer; draft_logits may be None when greedy).  The copies run
        on `copy_stream`, in the order the step consumes them, and every call waits only for
        its own inputs: the schedule starts once the confidences and lengths have landed, and
        layer i's attention overlaps the copy of layer i + 1's inputs.  The step's results
        (verify_len, accepted_len, out_tokens, n_out) are copied into `host_out` (pinned host
        tensors) on the current stream.  Returns the number of kernels launched."""
        cur = torch.cuda.current_stream(self.q_offsets.device)
        copy_stream.wait_stream(cur)  # the previous step is done with the device buffers
        layers = dev["q"].shape[0]
        e_sched, e_acc = torch.cuda.Event(), torch.cuda.Event()
        e_layer = [torch.cuda.Event() for _ in range(layers)]
        with torch.cuda.stream(copy_stream):
            for k in ("conf", "kv_len", "t_ms"):
                dev[k].copy_(host[k], non_blocking=True)
            e_sched.record(copy_stream)
            for i in range(layers):
                for k in ("q", "k_new", "v_new"):
                    dev[k][i].copy_(host[k][i], non_blocking=True)
                e_layer[i].record(copy_stream)
            for k in ("target_logits", "draft_logits", "draft_tokens", "u_acc", "u_res"):
                if host.get(k) is not None:
                    dev[k].copy_(host[k], non_blocking=True)
            e_acc.record(copy_stream)
        cur.wait_event(e_sched)
        self.schedule(dev["conf"], round_idx, dev["kv_len"], dev["t_ms"])
        self.plan(dev["kv_len"])
        for i in range(layers):
            cur.wait_event(e_layer[i])
            self.attention(dev["q"][i], dev["k_new"][i], dev["v_new"][i], kv_pages_per_layer[i],
                           block_table, dev["kv_len"], attn_out)
        cur.wait_event(e_acc)
        self.accept(dev["target_logits"], dev.get("draft_logits"), dev["draft_tokens"],
                    dev["u_acc"], dev["u_res"], temperature)
        if host_out is not None:
            for k in ("verify_len", "accepted_len", "out_tokens", "n_out"):
                host_out[k].copy_(getattr(self, k), non_blocking=True)
        return 2 + layers + 2

    def capture(self, enqueue, warmup: int = 1) -> torch.cuda.CUDAGraph:
        """Capture `enqueue()` — any sequence of this object's calls on the current stream — as
        one CUDA graph (after `warmup` eager runs on the capture stream).  Every launch is sized
        by capacities (R, K, T_cap, ...), never by device results, so the graph stays valid for
        whatever data the same buffers hold when it is replayed with `graph.replay()`."""
        dev = self.q_offsets.device
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for _ in range(warmup):
                enqueue()
        torch.cuda.current_stream(dev).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            enqueue()
        torch.cuda.current_stream(dev).wait_stream(s)
        return g

    def run(self, conf_ring, round_idx, kv_len, t_ms, layers, kv_pages_per_layer, block_table,
            attn_out, target_logits, draft_logits, draft_tokens, u_acc, u_res, temperature,
            stream=None) -> int:
        """Issue one whole step; `layers` is a sequence of (q, k_new, v_new) per layer and
        kv_pages_per_layer the matching caches.  Returns the number of kernels launched."""
        self.schedule(conf_ring, round_idx, kv_len, t_ms, stream)
        self.plan(kv_len, stream)
        for (q, k_new, v_new), kv in zip(layers, kv_pages_per_layer):
            self.attention(q, k_new, v_new, kv, block_table, kv_len, attn_out, stream)
        self.accept(target_logits, draft_logits, draft_tokens, u_acc, u_res, temperature, stream)
        return 2 + len(layers) + 2
