"""moe_layer_forward on the GPU against the oracle, for the tiny layer, the
GLM-scale decode layer (T=1), small batches with a Zipf-skewed router and a
4096-token prefill (sampled tokens).  Indices bit for bit except flagged
near-ties; max |y - y_ref| <= 2e-3 max |y_ref|."""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import GpuLayer, OracleLayer, flagged, rel_err, routing_is_valid

pytestmark = pytest.mark.gpu
TOL = 2e-3


def run_and_check(lib, L, OL, x, path=0, sample=None, bias=None):
    cfg = L.cfg
    T = x.shape[0]
    bias = L.bias if bias is None else bias
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(T, cfg.H, cfg.I, L.rcfg, path))
    y = lib.moe_layer_forward(x, L.gate, bias, L.rcfg, L.table, L.shared, L.bits, idx_out=idx,
                              w_out=w, ws=ws, path=path)
    assert ws.flags() == 0
    y, idx, w = y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    xb = syn.bf16_bits(x)
    if sample is not None:
        xb, y, idx, w = xb[sample], y[sample], idx[sample], w[sample]
    r = OL.route(xb)
    fl = flagged(r)
    assert np.array_equal(idx[~fl], r["idx"][~fl])
    assert np.allclose(w[~fl], r["w"][~fl], rtol=2e-6, atol=0)
    use_idx, use_w = r["idx"].copy(), r["w"].copy()
    for t in np.nonzero(fl)[0]:
        if not np.array_equal(idx[t], r["idx"][t]):
            assert routing_is_valid(r["scores"][t], OL.bias, idx[t], cfg)
            use_idx[t], use_w[t] = idx[t], w[t]
    ref = OL.layer_y(xb, use_idx, use_w)["y"]
    err = rel_err(y, ref)
    assert err <= TOL, err
    return err


@pytest.fixture(scope="module")
def tiny(lib):
    return GpuLayer(lib, syn.TINY)


@pytest.fixture(scope="module")
def tiny_orc(orc):
    return OracleLayer(orc, syn.TINY)


@pytest.mark.parametrize("T", [1, 4, 5, 33])
def test_layer_tiny(lib, tiny, tiny_orc, T):
    x = syn.activations(T, syn.TINY.H, T, "cuda")
    run_and_check(lib, tiny, tiny_orc, x)


def test_layer_empty_batch(lib, tiny):
    x = torch.empty((0, syn.TINY.H), dtype=torch.bfloat16, device="cuda")
    y = lib.moe_layer_forward(x, tiny.gate, tiny.bias, tiny.rcfg, tiny.table, tiny.shared, 4)
    assert y.shape == (0, syn.TINY.H)


def test_layer_tiny_no_shared(lib, tiny, orc):
    cfg = syn.TINY.with_(shared=False)
    L = GpuLayer(lib, cfg)
    OL = OracleLayer(orc, cfg)
    run_and_check(lib, L, OL, syn.activations(7, cfg.H, 70, "cuda"))


@pytest.fixture(scope="module")
def glm(lib):
    return GpuLayer(lib, syn.DECODE)


@pytest.fixture(scope="module")
def glm_orc(orc):
    return OracleLayer(orc, syn.DECODE)


@pytest.mark.parametrize("seed", [1, 2, 3, 9999])
def test_layer_glm_decode_t1(lib, glm, glm_orc, seed):
    run_and_check(lib, glm, glm_orc, syn.activations(1, syn.DECODE.H, seed, "cuda"))


@pytest.mark.parametrize("T", [2, 4, 8, 32])
def test_layer_glm_small_batch_zipf(lib, glm, orc, T):
    cfg = syn.SMALL_BATCH.with_(T=T)
    OL = OracleLayer(orc, cfg)
    bias = syn.router_bias(cfg, 0, "cuda")
    run_and_check(lib, glm, OL, syn.activations(T, cfg.H, 300 + T, "cuda"), bias=bias)


def test_layer_glm_prefill_sampled(lib, glm, glm_orc):
    x = syn.activations(4096, syn.DECODE.H, 4096, "cuda")
    rng = np.random.default_rng(4096)
    sample = np.sort(np.r_[0, 1, 4095, rng.choice(np.arange(2, 4095), 21, replace=False)])
    run_and_check(lib, glm, glm_orc, x, sample=sample)


def test_layer_deterministic(lib, glm):
    x = syn.activations(4, syn.DECODE.H, 77, "cuda")
    a = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4)
    b = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4)
    assert torch.equal(a, b)


def test_layer_accumulate_mode(lib, glm):
    x = syn.activations(2, syn.DECODE.H, 78, "cuda")
    a = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4)
    base = torch.full_like(a, 0.5)
    b = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              y=base.clone(), accumulate=True)
    assert torch.allclose(b, a + 0.5, rtol=0, atol=1e-5)
