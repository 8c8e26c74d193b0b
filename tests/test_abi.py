"""The C ABI library loads on any host and exports every entry point include/dspark.h declares.

Only host-side behaviour is exercised here (no kernel launches): symbol table, status strings,
version, workspace size queries that need no device, and argument validation that rejects a
call before anything is enqueued.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dspark.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from speculative_decoding_verification_survival_b200.build import build, LIB_PATH
    build()
    return ctypes.CDLL(LIB_PATH)


def test_header_declares_the_entry_points():
    names = _declared()
    for want in ("dspark_schedule", "dspark_verify_attn_plan", "dspark_verify_attn",
                 "dspark_accept", "dspark_read_error", "dspark_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_binding_covers_every_declared_symbol(lib):
    from speculative_decoding_verification_survival_b200 import dspark
    assert sorted(dspark.EXPORTED) == _declared()


def test_status_strings_and_version(lib):
    lib.dspark_status_string.restype = ctypes.c_char_p
    for code in (0, -1, -2, -3, -4, -5, -6):
        s = lib.dspark_status_string(code).decode()
        assert s.startswith("DSPARK_") and "UNKNOWN" not in s
    assert b"UNKNOWN" in lib.dspark_status_string(12345)
    assert lib.dspark_version() >= 100


def test_accept_workspace_query(lib):
    lib.dspark_accept_workspace_bytes.restype = ctypes.c_size_t
    assert lib.dspark_accept_workspace_bytes(64, 5, 384) == (384 + 64 * 5) * 16
    assert lib.dspark_accept_workspace_bytes(0, 5, 384) == 0
    assert lib.dspark_accept_workspace_bytes(64, 17, 384) == 0


def test_host_validation_rejects_before_launch(lib):
    from speculative_decoding_verification_survival_b200 import dspark as d
    f = lib.dspark_schedule
    f.argtypes = d._SIGS["dspark_schedule"][0]
    P = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    # NULL pointer
    assert f(None, 3, 0, 4, 5, P, P, 24, P, P, P, P, P, None) == -1
    # ring too shallow for the two-round lag
    assert f(P, 2, 0, 4, 5, P, P, 24, P, P, P, P, P, None) == -1
    # K above the supported maximum, T_cap below R
    assert f(P, 3, 0, 4, 17, P, P, 24, P, P, P, P, P, None) == -1
    assert f(P, 3, 0, 4, 5, P, P, 3, P, P, P, P, P, None) == -1
    # too many candidates for the one-CTA sort
    assert f(P, 3, 0, 4000, 5, P, P, 24000, P, P, P, P, P, None) == -6

    g = lib.dspark_verify_attn
    g.argtypes = d._SIGS["dspark_verify_attn"][0]
    args = [P, P, P, P, 10, P, 4, P, P, P, 4, 24, 8, 2, 128, 5, 64, 1, 0.1, P, P, 1 << 20, None]
    a = list(args); a[13] = 3                      # Hq % Hkv != 0
    assert g(*a) == -1
    a = list(args); a[14] = 100                    # D % 8 != 0
    assert g(*a) == -6
    a = list(args); a[12] = 64; a[13] = 2          # (Hq/Hkv)*(K+1) > 128
    assert g(*a) == -6
    a = list(args); a[17] = 7                      # unknown dtype
    assert g(*a) == -1
    a = list(args); a[0] = None
    assert g(*a) == -1

    h = lib.dspark_accept
    h.argtypes = d._SIGS["dspark_accept"][0]
    # sampled mode needs draft logits and uniforms
    assert h(P, None, 1, 32, 4, 5, 24, P, P, P, P, P, 1.0, P, P, P, P, 4096, None) == -1
    # workspace too small
    assert h(P, P, 1, 32, 4, 5, 24, P, P, P, P, P, 1.0, P, P, P, P, 8, None) == -3
    # NaN temperature
    assert h(P, P, 1, 32, 4, 5, 24, P, P, P, P, P, float("nan"), P, P, P, P, 4096, None) == -1


def test_kv_commit_host_validation(lib):
    from speculative_decoding_verification_survival_b200 import dspark as d
    f = lib.dspark_kv_commit
    f.argtypes = d._SIGS["dspark_kv_commit"][0]
    P, Q = ctypes.c_void_p(16), ctypes.c_void_p(32)
    base = [P, P, 0, P, 10, 0, 1, P, 4, P, P, P, 4, 24, 2, 128, 5, 64, 1, Q, None]
    a = list(base); a[19] = P                       # kv_len_out aliases kv_len
    assert f(*a) == -1
    a = list(base); a[18] = 9                       # unknown dtype
    assert f(*a) == -1
    a = list(base); a[15] = 4                       # D * 2 bytes not a multiple of 16
    assert f(*a) == -1
    a = list(base); a[6] = 2                        # two layers with no layer stride
    assert f(*a) == -1
    a = list(base); a[0] = ctypes.c_void_p(18)      # misaligned k_new
    assert f(*a) == -1
    a = list(base); a[16] = 17                      # K above the supported maximum
    assert f(*a) == -1
