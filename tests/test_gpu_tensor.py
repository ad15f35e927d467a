"""The tcgen05 tensor-core path of moe_layer_forward against the oracle:
tiny and GLM-scale layers, ragged token counts, experts with more tokens than
one tile (Zipf-skewed router), and agreement with the CUDA-core path."""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import GpuLayer, OracleLayer, rel_err
from test_gpu_layer import run_and_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny(lib):
    return GpuLayer(lib, syn.TINY)


@pytest.fixture(scope="module")
def tiny_orc(orc):
    return OracleLayer(orc, syn.TINY)


@pytest.mark.parametrize("T", [1, 5, 64, 300])
def test_tensor_path_tiny(lib, tiny, tiny_orc, T):
    x = syn.activations(T, syn.TINY.H, 1000 + T, "cuda")
    run_and_check(lib, tiny, tiny_orc, x, path=lib.PATH_TENSOR)


@pytest.fixture(scope="module")
def glm(lib):
    return GpuLayer(lib, syn.DECODE)


@pytest.fixture(scope="module")
def glm_orc(orc):
    return OracleLayer(orc, syn.DECODE)


@pytest.mark.parametrize("T", [16, 200])
def test_tensor_path_glm(lib, glm, glm_orc, T):
    run_and_check(lib, glm, glm_orc, syn.activations(T, syn.DECODE.H, 2000 + T, "cuda"),
                  path=lib.PATH_TENSOR)


def test_tensor_path_glm_zipf_many_tokens_per_expert(lib, glm, orc):
    """Zipf bias routes several hundred tokens to hot experts (several tiles)."""
    cfg = syn.SMALL_BATCH.with_(T=1024)
    OL = OracleLayer(orc, cfg)
    bias = syn.router_bias(cfg, 0, "cuda")
    x = syn.activations(1024, cfg.H, 3001, "cuda")
    idx, _, _ = lib.moe_route_topk(x, glm.gate, bias, glm.rcfg)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=cfg.E)
    assert counts.max() > 128
    sample = np.r_[0:8, np.random.default_rng(5).choice(1024, 12, replace=False)]
    run_and_check(lib, glm, OL, x, path=lib.PATH_TENSOR, sample=np.unique(sample), bias=bias)


def test_tensor_and_gemv_paths_agree(lib, glm):
    x = syn.activations(96, syn.DECODE.H, 4001, "cuda")
    a = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              path=lib.PATH_TENSOR)
    b = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              path=lib.PATH_GEMV)
    assert rel_err(a.cpu().numpy(), b.cpu().numpy()) <= 2e-3


def test_tensor_path_accumulates(lib, glm):
    x = syn.activations(64, syn.DECODE.H, 4002, "cuda")
    a = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              path=lib.PATH_TENSOR)
    base = torch.full_like(a, -0.25)
    b = lib.moe_layer_forward(x, glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              y=base.clone(), accumulate=True, path=lib.PATH_TENSOR)
    assert torch.allclose(b, a - 0.25, rtol=0, atol=1e-4)


def test_tensor_path_bitwise_reproducible(lib, glm):
    """Per-pair partials combined in a fixed order: identical y run to run,
    including experts that span several token tiles."""
    cfg = syn.SMALL_BATCH.with_(T=1024)
    bias = syn.router_bias(cfg, 0, "cuda")
    x = syn.activations(1024, cfg.H, 3002, "cuda")
    a = lib.moe_layer_forward(x, glm.gate, bias, glm.rcfg, glm.table, glm.shared, 4,
                              path=lib.PATH_TENSOR)
    b = lib.moe_layer_forward(x, glm.gate, bias, glm.rcfg, glm.table, glm.shared, 4,
                              path=lib.PATH_TENSOR)
    assert torch.equal(a, b)
