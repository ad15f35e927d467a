"""moe_route_topk on the GPU against the oracle: indices bit for bit except on
tokens whose decision margin is below 1e-6 (checked as valid selections),
weights to 1e-6 relative, for the tiny and GLM-scale router configurations
and random tiny group layouts."""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import flagged, routing_is_valid

pytestmark = pytest.mark.gpu


def _check(lib, orc, cfg, T, seed, gate, bias):
    x = syn.activations(T, cfg.H, seed, "cuda")
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
    idx, w, gap = lib.moe_route_topk(x, gate, bias, rc, with_gap=True)
    xb = syn.bf16_bits(x)
    r = orc.route(xb, gate.cpu().numpy(), bias.cpu().numpy(), cfg.k, cfg.n_group,
                  cfg.topk_group, cfg.rsf, cfg.topp)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    fl = flagged(r)
    ok = ~fl
    assert np.array_equal(idx[ok], r["idx"][ok])
    assert np.allclose(w[ok], r["w"][ok], rtol=1e-6, atol=0)
    for t in np.nonzero(fl)[0]:
        if not np.array_equal(idx[t], r["idx"][t]):
            assert routing_is_valid(r["scores"][t], bias.cpu().numpy(), idx[t], cfg), t
    g = gap.cpu().numpy()
    want = np.minimum(r["gap"], r["ggap"])
    fin = np.isfinite(want)
    assert np.all(np.isinf(g[~fin]))
    assert np.allclose(g[fin], want[fin], rtol=1e-3, atol=1e-6)
    return int(fl.sum())


def test_router_tiny(lib, orc):
    cfg = syn.TINY
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    for seed in range(8):
        _check(lib, orc, cfg, cfg.T, seed, gate, bias)


@pytest.mark.parametrize("T", [1, 3, 8, 64, 65, 300])
def test_router_glm_scale(lib, orc, T):
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    _check(lib, orc, cfg, T, 100 + T, gate, bias)


def test_router_glm_zipf_bias(lib, orc):
    cfg = syn.SMALL_BATCH
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    for T in (2, 4, 8, 32):
        _check(lib, orc, cfg.with_(T=T), T, 200 + T, gate, bias)


def test_router_many_decode_tokens(lib, orc):
    """2000 single-token calls' worth of tokens (fresh seeds), decode kernel."""
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    for chunk in range(40):
        _check(lib, orc, cfg, 50, 10_000 + chunk, gate, bias)


@pytest.mark.parametrize("E,n_group,topk_group,k", [(8, 1, 1, 2), (12, 3, 2, 4), (12, 2, 1, 3),
                                                    (9, 3, 3, 9), (64, 4, 2, 6), (1024, 32, 4, 8)])
def test_router_group_layouts(lib, orc, E, n_group, topk_group, k):
    cfg = syn.LayerConfig("t", H=128, I=64, E=E, k=k, n_group=n_group, topk_group=topk_group,
                          rsf=2.5, bias_amp=0.1)
    gate = syn.normal((E, 128), 0.3, E * 31 + k, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    _check(lib, orc, cfg, 40, E + k, gate, bias)


def test_router_expert_topp(lib, orc):
    cfg = syn.DECODE.with_(topp=0.7)
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    _check(lib, orc, cfg, 64, 7, gate, bias)


def test_router_prefill_sample(lib, orc):
    """4096 tokens through the tiled logits kernel; the oracle checks a sample."""
    cfg = syn.PREFILL
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    x = syn.activations(4096, cfg.H, 4242, "cuda")
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf)
    idx, w, _ = lib.moe_route_topk(x, gate, bias, rc)
    sample = np.r_[0:64, 4000:4096, np.random.default_rng(0).choice(4096, 96, replace=False)]
    xb = syn.bf16_bits(x)[sample]
    r = orc.route(xb, gate.cpu().numpy(), bias.cpu().numpy(), cfg.k, cfg.n_group,
                  cfg.topk_group, cfg.rsf)
    idx, w = idx.cpu().numpy()[sample], w.cpu().numpy()[sample]
    ok = ~flagged(r)
    assert np.array_equal(idx[ok], r["idx"][ok])
    assert np.allclose(w[ok], r["w"][ok], rtol=2e-6, atol=0)
