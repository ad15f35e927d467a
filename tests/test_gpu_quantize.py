"""moe_quantize_rows on the GPU against the oracle: packed bytes and scales
bit for bit (bits 4, 8, 2), ragged sizes, hand-made ties, zero rows."""
import numpy as np
import pytest
import torch

from golden_io import rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [4, 8, 2])
@pytest.mark.parametrize("shape", [(1, 64), (37, 256), (130, 132), (8, 6144), (1000, 2048)])
def test_quantize_bit_exact(lib, orc, bits, shape):
    R, C = shape
    if bits == 2 and C % 4:
        C += 4 - C % 4
    rng = np.random.default_rng(R * 7 + C + bits)
    w = (rng.standard_normal((R, C)) * 0.02).astype(np.float32)
    w[0, :] = 0.0
    if R > 3:
        w[2, ::3] = np.float32(-0.03)
        w[3, :] = np.float32(1e-30)  # tiny but normal-range scale
    q, s = lib.moe_quantize_rows(torch.from_numpy(w).cuda(), bits)
    qo, so = orc.quantize_rows(w, bits)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), qo)


def test_quantize_golden_rows(lib, orc):
    for bits, vals, scale, codes in rows("quantize_rows.txt"):
        bits = int(bits)
        w = np.array([[float(v) for v in vals.split()]], np.float32)
        q, s = lib.moe_quantize_rows(torch.from_numpy(w).cuda(), bits)
        assert float(s.item()) == float(np.float32(float(scale)))
        got = orc.unpack(q.cpu().numpy(), w.shape[1], bits)[0].tolist()
        assert got == [int(c) for c in codes.split()], (bits, vals)


def test_quantize_glm_expert_matrix(lib, orc):
    from int4_routed_expert_route_b200 import synthetic as syn
    cfg = syn.DECODE
    for m in ("gate", "down"):
        w = syn.expert_weight(cfg, 0, 3, m, "cuda")
        q, s = lib.moe_quantize_rows(w, 4)
        qo, so = orc.quantize_rows(w.cpu().numpy(), 4)
        assert np.array_equal(q.cpu().numpy(), qo)
        assert np.array_equal(s.cpu().numpy(), so)
