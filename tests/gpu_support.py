"""Helpers for GPU parity tests: run the CUDA path and the oracle on identical input bits.

Inputs come from workloads/ (seeded); the oracle reads back exactly the tensors the GPU got
(bf16 values upcast exactly).  No expected value is ever taken from the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle.schedule import lagged_round
from workloads.generate import flatten_target

ATTN_MAX_ABS = 2e-2   # stated tolerance for bf16 attention outputs
ATTN_MEAN_ABS = 2e-3
F32_ATTN_MAX_ABS = 1e-4


def binding():
    from speculative_decoding_verification_survival_b200 import dspark
    return dspark


def new_step(cfg, device="cuda"):
    from speculative_decoding_verification_survival_b200 import VerifyStep
    return VerifyStep(cfg.R, cfg.K, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, device=device)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def gpu_schedule(step, inp):
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    torch.cuda.synchronize()
    T = int(step.T.item())
    return dict(verify_len=host(step.verify_len), q_offsets=host(step.q_offsets),
                markers=host(step.markers)[:T], T=T, objective=float(step.objective.item()))


def oracle_schedule(inp):
    conf = inp.conf_history[lagged_round(inp.round_idx)]
    return oracle.schedule_ref(conf, host(inp.kv_len), host(inp.t_ms), inp.cfg.T_cap)


def assert_schedule_equal(gpu, ref):
    if ref["flagged"]:
        return 1
    assert np.array_equal(gpu["verify_len"], ref["verify_len"])
    assert np.array_equal(gpu["q_offsets"], ref["q_offsets"])
    assert gpu["T"] == ref["T"]
    assert np.array_equal(gpu["markers"], ref["markers"])
    assert math.isclose(gpu["objective"], ref["objective"], rel_tol=1e-12)
    return 0


def set_schedule(step, verify_len, kv_len):
    """Install a chosen schedule (from the oracle's flattening) into the step's buffers."""
    qo, mk = oracle.flatten_ref(verify_len, kv_len)
    dev = step.verify_len.device
    step.verify_len.copy_(torch.as_tensor(np.asarray(verify_len, np.int32)).to(dev))
    step.q_offsets.copy_(torch.as_tensor(qo).to(dev))
    step.markers.zero_()
    step.markers[:len(mk)] = torch.as_tensor(mk).to(dev)
    step.T.fill_(int(qo[-1]))
    return qo, mk


def oracle_attn_rows(inp, layer, cache, qo, mk, rows, scale):
    """Oracle attention for the listed flat (t, h) rows, reading only the touched requests'
    pages from the device cache."""
    cfg = inp.cfg
    kv = host(inp.kv_len)
    table = host(inp.block_table)
    by_req = {}
    for t, h in rows:
        by_req.setdefault(int(mk[t, 0]), []).append((t, h))
    out = {}
    for r, rr in by_req.items():
        n = int(kv[r])
        npg = max(1, -(-n // cfg.page_size))
        pages = torch.as_tensor(table[r, :npg].astype(np.int64), device=cache.device)
        local = host(cache.index_select(0, pages))
        t0, t1 = int(qo[r]), int(qo[r + 1])
        res = oracle.attn_ref_flat(
            host(inp.q[layer, t0:t1]), host(inp.k_new[layer, t0:t1]), host(inp.v_new[layer, t0:t1]),
            local, np.arange(npg, dtype=np.int32)[None, :], np.array([n]),
            np.stack([np.zeros(t1 - t0, np.int32), mk[t0:t1, 1]], axis=1),
            np.array([0, t1 - t0]), scale, cfg.page_size,
            rows=[(t - t0, h) for t, h in rr])
        for t, h in rr:
            out[(t, h)] = res[t - t0, h]
    return out


def oracle_accept_chunked(target_flat, draft_logits, draft_tokens, verify_len, q_offsets, u_acc,
                          u_res, temperature, chunk=32):
    """accept_ref over request chunks, copying only the rows each chunk needs."""
    R = draft_tokens.shape[0]
    qo = np.asarray(q_offsets)
    outs = []
    for r0 in range(0, R, chunk):
        r1 = min(R, r0 + chunk)
        t0, t1 = int(qo[r0]), int(qo[r1])
        res = oracle.accept_ref(
            host(target_flat[t0:t1]),
            host(draft_logits[r0:r1]) if temperature > 0 else np.zeros((r1 - r0, 1, 1)),
            draft_tokens[r0:r1], verify_len[r0:r1], qo[r0:r1 + 1] - t0,
            u_acc[r0:r1], u_res[r0:r1], temperature)
        outs.append(res)
    return {k: np.concatenate([o[k] for o in outs]) for k in outs[0]}


def assert_accept_equal(gpu, ref):
    """Bit-exact on every unflagged request; returns (#flagged, #flagged that differ)."""
    same = ((gpu["accepted_len"] == ref["accepted_len"])
            & np.all(gpu["out_tokens"] == ref["out_tokens"], axis=1)
            & (gpu["n_out"] == ref["n_out"]))
    bad = ~same & ~ref["flagged"]
    assert not np.any(bad), (f"{int(bad.sum())} unflagged requests differ, first "
                             f"{np.nonzero(bad)[0][:5].tolist()}")
    return int(ref["flagged"].sum()), int((~same & ref["flagged"]).sum())


def gpu_accept(step, target_flat, draft_logits, draft_tokens, u_acc, u_res, temperature):
    step.accept(target_flat, draft_logits if temperature > 0 else None, draft_tokens,
                u_acc, u_res, temperature)
    torch.cuda.synchronize()
    return dict(accepted_len=host(step.accepted_len), out_tokens=host(step.out_tokens),
                n_out=host(step.n_out))


def flat_target(inp, verify_len):
    return flatten_target(inp.target_block, verify_len, inp.cfg.T_cap)
