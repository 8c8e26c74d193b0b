"""Philox4x32-10 input generator against its published known-answer vectors."""
import os

import numpy as np

from workloads.philox import philox4x32, step_uniforms, uniforms_from_words

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    with open(GOLDEN) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            w = [int(x, 16) for x in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_known_answer_vectors():
    rows = _kat()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = philox4x32(np.array(ctr, dtype=np.uint32), np.array(key, dtype=np.uint32))
        assert [int(v) for v in got] == want


def test_vectorised_matches_scalar():
    ctr = np.array([[i, 7 * i, 3, 11] for i in range(50)], dtype=np.uint32)
    key = np.array([5, 9], dtype=np.uint32)
    batch = philox4x32(ctr, key)
    for i in range(50):
        assert np.array_equal(batch[i], philox4x32(ctr[i], key))


def test_uniform_convention():
    w = np.array([0, 0xFF, 0x100, 0xFFFFFFFF], dtype=np.uint32)
    u = uniforms_from_words(w)
    assert u.dtype == np.float32
    assert u[0] == 0.0 and u[1] == 0.0
    assert u[2] == np.float32(2.0 ** -24)
    assert u[3] == np.float32(1.0 - 2.0 ** -24) and u[3] < 1.0


def test_step_uniform_shapes_and_independence():
    ua, ur = step_uniforms(3, 17, 5)
    assert ua.shape == (17, 5) and ur.shape == (17, 6)
    assert np.all((ua >= 0) & (ua < 1)) and np.all((ur >= 0) & (ur < 1))
    ua2, _ = step_uniforms(4, 17, 5)
    assert not np.array_equal(ua, ua2)
    big, _ = step_uniforms(0, 20000, 5)
    assert abs(big.mean() - 0.5) < 0.01
