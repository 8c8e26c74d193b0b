"""Thin ctypes binding of libdspark (include/dspark.h): argument marshalling only.

Every function below has the name of the C entry point it calls and forwards device pointers
of caller-provided torch tensors plus the current CUDA stream.  Nothing here computes any part
of the verify step; if the shared library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

DSPARK_OK = 0
DSPARK_F32 = 0
DSPARK_BF16 = 1
DSPARK_CONF_LAG = 2
DSPARK_MAX_K = 16
DSPARK_MAX_CANDIDATES = 16384
DSPARK_ACCEPT_NOALLOC_MAX_ROWS = 65536

DEVICE_ERROR_BITS = {
    1 << 0: "CONF", 1 << 1: "TABLE", 1 << 2: "KV_LEN", 1 << 3: "PAGE", 1 << 4: "MARKER",
    1 << 5: "OFFSETS", 1 << 6: "VERIFY_LEN", 1 << 7: "TOKEN", 1 << 8: "LOGITS",
    1 << 9: "TIMEOUT", 1 << 10: "ACCEPTED",
}


class DSparkError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = _lib.dspark_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdspark.so is not built ({LIB_PATH}); run "
                          "speculative_decoding_verification_survival_b200.build.build()")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()
_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGS = {
    "dspark_status_string": ([_i], ctypes.c_char_p),
    "dspark_version": ([], _i),
    "dspark_schedule": ([_p, _i, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p], _i),
    "dspark_flatten_markers": ([_p, _p, _i, _i, _i, _p, _p], _i),
    "dspark_verify_attn_workspace_bytes": ([_i, _i, _i, _i, _i], _sz),
    "dspark_verify_attn_plan": ([_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _sz, _p], _i),
    "dspark_verify_attn": ([_p, _p, _p, _p, _i64, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                            _i, _i, _f, _p, _p, _sz, _p], _i),
    "dspark_accept_workspace_bytes": ([_i, _i, _i], _sz),
    "dspark_accept": ([_p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _f, _p, _p, _p, _p, _sz,
                       _p], _i),
    "dspark_read_error": ([ctypes.POINTER(ctypes.c_int32), _p], _i),
    "dspark_selftest_wait_timeout": ([ctypes.c_longlong, _p, _p], _i),
    "dspark_markov_draft_workspace_bytes": ([_i, _i], _sz),
    "dspark_markov_draft": ([_p, _p, _p, _i, _p, _i, _i, _i, _f, ctypes.c_uint32, ctypes.c_uint32,
                             _p, _p, _p, _sz, _p], _i),
    "dspark_calibrate_confidence": ([_p, _p, _i, _i, _p, _p], _i),
    "dspark_fit_temperature": ([_p, _p, _p, _i, _i, _p, _p], _i),
    "dspark_kv_commit": ([_p, _p, _i64, _p, _i64, _i64, _i, _p, _i, _p, _p, _p, _i, _i, _i, _i,
                          _i, _i, _i, _p, _p], _i),
    "dspark_accept_noalloc": ([_p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _f, _p, _p, _p,
                               _p], _i),
}
for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _ret

EXPORTED = tuple(_SIGS)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensors passed to libdspark must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libdspark must be contiguous")
    return t.data_ptr()


def _check(t, dtype, name):
    if t is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _call(name, *args):
    st = getattr(_lib, name)(*args)
    if st != DSPARK_OK:
        raise DSparkError(name, st)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSPARK_BF16
    if t.dtype == torch.float32:
        return DSPARK_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def dspark_version() -> int:
    return _lib.dspark_version()


def dspark_status_string(status: int) -> str:
    return _lib.dspark_status_string(status).decode()


def dspark_schedule(conf_ring, round_idx, kv_len, t_ms, T_cap, verify_len, q_offsets, markers,
                    T_out, objective, stream=None):
    """conf_ring float32 [depth][R][K]; kv_len int32 [R]; t_ms float64 [T_cap+1];
    outputs verify_len int32 [R], q_offsets int32 [R+1], markers int32 [T_cap][2],
    T_out int32 [1], objective float64 [1].  kv_len = markers = None: lengths only."""
    depth, R, K = conf_ring.shape
    _check(conf_ring, torch.float32, "conf_ring")
    _check(kv_len, torch.int32, "kv_len")
    _check(t_ms, torch.float64, "t_ms")
    _call("dspark_schedule", _ptr(conf_ring), depth, int(round_idx), R, K, _ptr(kv_len),
          _ptr(t_ms), int(T_cap), _ptr(verify_len), _ptr(q_offsets), _ptr(markers), _ptr(T_out),
          _ptr(objective), _stream(stream))


def dspark_flatten_markers(kv_len, q_offsets, K, markers, stream=None):
    """kv_len int32 [R]; q_offsets int32 [R+1] (from a lengths-only schedule); markers out
    int32 [T_cap][2]."""
    for t, n in ((kv_len, "kv_len"), (q_offsets, "q_offsets"), (markers, "markers")):
        _check(t, torch.int32, n)
    _call("dspark_flatten_markers", _ptr(kv_len), _ptr(q_offsets), kv_len.shape[0], int(K),
          markers.shape[0], _ptr(markers), _stream(stream))


def dspark_verify_attn_workspace_bytes(R, Hq, Hkv, D, K) -> int:
    return int(_lib.dspark_verify_attn_workspace_bytes(R, Hq, Hkv, D, K))


def dspark_verify_attn_plan(kv_len, q_offsets, markers, R, Hq, Hkv, D, K, ws, stream=None):
    """kv_len int32 [R]; q_offsets int32 [R + 1]; markers int32 [T_cap][2]."""
    for t, n in ((kv_len, "kv_len"), (q_offsets, "q_offsets"), (markers, "markers")):
        _check(t, torch.int32, n)
    _call("dspark_verify_attn_plan", _ptr(kv_len), _ptr(q_offsets), _ptr(markers), R,
          markers.shape[0], Hq, Hkv, D, K, _ptr(ws), ws.numel(), _stream(stream))


def dspark_verify_attn(q, k_new, v_new, kv_pages, block_table, kv_len, markers, q_offsets, K,
                       scale, out, ws, stream=None):
    """q [T_cap][Hq][D]; k_new/v_new [T_cap][Hkv][D]; kv_pages [P][2][Hkv][page][D];
    block_table int32 [R][max_pages]; out [T_cap][Hq][D]."""
    T_cap, Hq, D = q.shape
    Hkv = k_new.shape[1]
    num_pages, _, _, page_size, _ = kv_pages.shape
    R, max_pages = block_table.shape
    for t in (k_new, v_new, kv_pages, out):
        if t.dtype != q.dtype:
            raise TypeError("q, k_new, v_new, kv_pages and out must share a dtype")
    _call("dspark_verify_attn", _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kv_pages), num_pages,
          _ptr(block_table), max_pages, _ptr(kv_len), _ptr(markers), _ptr(q_offsets), R, T_cap,
          Hq, Hkv, D, int(K), page_size, _dtype_code(q), float(scale), _ptr(out), _ptr(ws),
          ws.numel(), _stream(stream))


def dspark_accept_workspace_bytes(R, K, T_cap) -> int:
    return int(_lib.dspark_accept_workspace_bytes(R, K, T_cap))


def dspark_accept(target_logits, draft_logits, draft_tokens, verify_len, q_offsets, u_acc, u_res,
                  temperature, accepted_len, out_tokens, n_out, ws, stream=None):
    """target_logits [T_cap][V]; draft_logits [R][K][V] (None allowed when greedy);
    draft_tokens int32 [R][K]; u_acc float32 [R][K]; u_res float32 [R][K+1]."""
    T_cap, V = target_logits.shape
    R, K = draft_tokens.shape
    if draft_logits is not None and draft_logits.dtype != target_logits.dtype:
        raise TypeError("target and draft logits must share a dtype")
    _call("dspark_accept", _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits),
          V, R, K, T_cap, _ptr(draft_tokens), _ptr(verify_len), _ptr(q_offsets), _ptr(u_acc),
          _ptr(u_res), float(temperature), _ptr(accepted_len), _ptr(out_tokens), _ptr(n_out),
          _ptr(ws), ws.numel(), _stream(stream))


def dspark_read_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    _call("dspark_read_error", ctypes.byref(code), _stream(stream))
    return int(code.value)


def decode_device_error(code: int):
    return [name for bit, name in DEVICE_ERROR_BITS.items() if code & bit]


def dspark_accept_noalloc(target_logits, draft_logits, draft_tokens, verify_len, q_offsets, u_acc,
                          u_res, temperature, accepted_len, out_tokens, n_out, stream=None):
    """dspark_accept without a workspace argument, for callers that cannot allocate device
    memory: the scratch is a fixed array inside the library (see include/dspark.h)."""
    T_cap, V = target_logits.shape
    R, K = draft_tokens.shape
    if draft_logits is not None and draft_logits.dtype != target_logits.dtype:
        raise TypeError("target and draft logits must share a dtype")
    _call("dspark_accept_noalloc", _ptr(target_logits), _ptr(draft_logits),
          _dtype_code(target_logits), V, R, K, T_cap, _ptr(draft_tokens), _ptr(verify_len),
          _ptr(q_offsets), _ptr(u_acc), _ptr(u_res), float(temperature), _ptr(accepted_len),
          _ptr(out_tokens), _ptr(n_out), _stream(stream))


def dspark_kv_commit(k_new, v_new, kv_pages, block_table, kv_len, q_offsets, accepted_len, K,
                     kv_len_out, stream=None):
    """Kept verify rows into the paged cache.  k_new / v_new [layers][T_cap][Hkv][D] (or
    [T_cap][Hkv][D] for one layer); kv_pages [layers][P][2][Hkv][page][D] (or one cache);
    kv_len_out int32 [R] must not alias kv_len."""
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(0), v_new.unsqueeze(0)
    if kv_pages.dim() == 5:
        kv_pages = kv_pages.unsqueeze(0)
    layers, T_cap, Hkv, D = k_new.shape
    if kv_pages.shape[0] != layers or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new and kv_pages must have the same number of layers")
    _, num_pages, _, _, page_size, _ = kv_pages.shape
    R, max_pages = block_table.shape
    for t in (v_new, kv_pages):
        if t.dtype != k_new.dtype:
            raise TypeError("k_new, v_new and kv_pages must share a dtype")
    for t, n in ((block_table, "block_table"), (kv_len, "kv_len"), (q_offsets, "q_offsets"),
                 (accepted_len, "accepted_len"), (kv_len_out, "kv_len_out")):
        _check(t, torch.int32, n)
    _call("dspark_kv_commit", _ptr(k_new), _ptr(v_new), k_new[0].numel(), _ptr(kv_pages),
          num_pages, kv_pages[0].numel(), layers, _ptr(block_table), max_pages, _ptr(kv_len),
          _ptr(q_offsets), _ptr(accepted_len), R, T_cap, Hkv, D, int(K), page_size,
          _dtype_code(k_new), _ptr(kv_len_out), _stream(stream))


def dspark_calibrate_confidence(logits, tau, conf, stream=None):
    """conf[r][k] = sigmoid(logits[r][k] / tau[k]); logits / conf float32 [R][K] (conf may be a
    slot of the confidence ring), tau float32 [K]."""
    R, K = logits.shape
    for t, n in ((logits, "logits"), (tau, "tau"), (conf, "conf")):
        _check(t, torch.float32, n)
    if tuple(conf.shape) != (R, K) or tau.numel() != K:
        raise ValueError("logits, conf must be [R][K] and tau [K]")
    _call("dspark_calibrate_confidence", _ptr(logits), _ptr(tau), R, K, _ptr(conf),
          _stream(stream))


def dspark_fit_temperature(logits, verify_len, accepted_len, tau, stream=None):
    """Maximum-likelihood per-position temperatures from N verified requests' raw confidence
    logits [N][K] (float32), verify_len / accepted_len int32 [N]; writes tau float32 [K]."""
    N, K = logits.shape
    _check(logits, torch.float32, "logits")
    _check(tau, torch.float32, "tau")
    _check(verify_len, torch.int32, "verify_len")
    _check(accepted_len, torch.int32, "accepted_len")
    _call("dspark_fit_temperature", _ptr(logits), _ptr(verify_len), _ptr(accepted_len), N, K,
          _ptr(tau), _stream(stream))


def dspark_markov_draft_workspace_bytes(R, V) -> int:
    return int(_lib.dspark_markov_draft_workspace_bytes(R, V))


def dspark_markov_draft(block_logits, E, U, x0, temperature, round_idx, seed, draft_logits,
                        draft_tokens, ws, stream=None):
    """Synthetic Markov-head draft: block_logits bf16 [R][K][V], E bf16 [V][d], U bf16 [d][V],
    x0 int32 [R]; writes draft_logits bf16 [R][K][V] and draft_tokens int32 [R][K]."""
    R, K, V = block_logits.shape
    d = E.shape[1]
    for t, n in ((block_logits, "block_logits"), (E, "E"), (U, "U"), (draft_logits, "draft_logits")):
        _check(t, torch.bfloat16, n)
    _check(x0, torch.int32, "x0")
    _check(draft_tokens, torch.int32, "draft_tokens")
    if tuple(U.shape) != (d, V) or E.shape[0] != V or tuple(draft_logits.shape) != (R, K, V):
        raise ValueError("shapes: block_logits [R][K][V], E [V][d], U [d][V], draft_logits [R][K][V]")
    _call("dspark_markov_draft", _ptr(block_logits), _ptr(E), _ptr(U), d, _ptr(x0), R, K, V,
          float(temperature), int(round_idx) & 0xFFFFFFFF, int(seed) & 0xFFFFFFFF,
          _ptr(draft_logits), _ptr(draft_tokens), _ptr(ws), ws.numel(), _stream(stream))


def dspark_selftest_wait_timeout(limit_cycles: int, result, stream=None):
    """A bounded in-kernel wait on a barrier nothing arrives at; result int32 [2] (device)."""
    _check(result, torch.int32, "result")
    _call("dspark_selftest_wait_timeout", int(limit_cycles), _ptr(result), _stream(stream))
