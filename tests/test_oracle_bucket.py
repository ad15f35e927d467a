"""Pins for the oracle's batch-union bucketing (a stable counting sort)."""
import numpy as np


def test_bucket_equals_stable_sort(orc):
    rng = np.random.default_rng(21)
    for T, k, E in [(1, 8, 256), (7, 2, 8), (64, 8, 256), (300, 4, 16)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        b = orc.bucket(idx, E)
        flat = idx.reshape(-1)
        order = sorted(range(T * k), key=lambda p: (flat[p], p))
        assert b["list"].tolist() == order
        assert np.array_equal(b["counts"], np.bincount(flat, minlength=E))
        assert b["offsets"][0] == 0 and np.array_equal(np.diff(b["offsets"]), b["counts"])
        assert b["unique"].tolist() == sorted(set(flat.tolist()))


def test_bucket_skips_dropped_pairs(orc):
    idx = np.array([[2, -1], [-1, 0], [2, 0]], np.int32)
    b = orc.bucket(idx, 4)
    assert b["list"].tolist() == [3, 5, 0, 4]
    assert b["counts"].tolist() == [2, 0, 2, 0]
    assert b["unique"].tolist() == [0, 2]
