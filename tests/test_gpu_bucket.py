"""moe_bucket on the GPU against the oracle's stable counting sort (bit exact)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 2, 8), (32, 8, 256), (4096, 8, 256),
                                   (777, 5, 1024), (3000, 1, 3)])
def test_bucket_bit_exact(lib, orc, T, k, E):
    rng = np.random.default_rng(T + k + E)
    if k <= E:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    else:
        idx = rng.integers(0, E, (T, k)).astype(np.int32)
    idx[rng.random((T, k)) < 0.05] = -1  # pairs dropped by expert top-p
    out = lib.moe_bucket(torch.from_numpy(idx).cuda(), E)
    ref = orc.bucket(idx, E)
    n = int(ref["offsets"][E])
    assert np.array_equal(out["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(out["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(out["list"].cpu().numpy()[:n], ref["list"])
    nu = int(out["n_unique"].item())
    assert nu == len(ref["unique"])
    assert np.array_equal(out["unique"].cpu().numpy()[:nu], ref["unique"])


def test_bucket_empty_batch(lib):
    out = lib.moe_bucket(torch.empty((0, 8), dtype=torch.int32, device="cuda"), 256)
    assert int(out["n_unique"].item()) == 0
    assert int(out["offsets"][-1].item()) == 0
