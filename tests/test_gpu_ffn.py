"""moe_expert_ffn on the GPU against the oracle (max |dy| <= 2e-3 max |y_ref|)."""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import OracleLayer, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _expert(lib, cfg, e, bits):
    w = [syn.expert_weight(cfg, 0, e, m, "cuda") for m in ("gate", "up", "down")]
    return lib.QuantExpert.from_fp32(*w, bits=bits)


@pytest.mark.parametrize("bits", [4, 8, 2])
@pytest.mark.parametrize("cfg", [syn.TINY, syn.DECODE], ids=["tiny", "glm"])
def test_expert_ffn_all_rows(lib, orc, cfg, bits):
    T = 3
    ex = _expert(lib, cfg, 1, bits)
    x = syn.activations(T, cfg.H, 5, "cuda")
    y = torch.zeros((T, cfg.H), dtype=torch.float32, device="cuda")
    lib.moe_expert_ffn(x, ex, y)
    ref = orc.expert_ffn(syn.bf16_bits(x), OracleLayer(orc, cfg, bits=bits).expert(1), cfg.H, cfg.I)
    assert rel_err(y.cpu().numpy(), ref) <= TOL


def test_expert_ffn_row_subset_accumulates(lib, orc):
    cfg = syn.DECODE
    ex = _expert(lib, cfg, 2, 4)
    T = 6
    x = syn.activations(T, cfg.H, 6, "cuda")
    rows = torch.tensor([4, 1, 5], dtype=torch.int32, device="cuda")
    rw = torch.tensor([0.5, -2.0, 1.25], dtype=torch.float32, device="cuda")
    base = torch.randn((T, cfg.H), generator=torch.Generator("cuda").manual_seed(1),
                       device="cuda")
    y = base.clone()
    lib.moe_expert_ffn(x, ex, y, rows=rows, row_w=rw)
    ref = orc.expert_ffn(syn.bf16_bits(x), OracleLayer(orc, cfg).expert(2), cfg.H, cfg.I)
    want = base.cpu().numpy().astype(np.float64)
    for r, wgt in zip([4, 1, 5], [0.5, -2.0, 1.25]):
        want[r] += wgt * ref[r]
    got = y.cpu().numpy()
    assert np.array_equal(got[[0, 2, 3]], base.cpu().numpy()[[0, 2, 3]])
    assert rel_err(got - base.cpu().numpy(), want - base.cpu().numpy().astype(np.float64)) <= TOL
