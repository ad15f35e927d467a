"""moe_layer_forward at full size and on its small-batch routing kernels,
against the oracle.

The small-batch paths select experts inside their own kernels (the fused router
for one or two tokens, the fused decode kernel for 3..8 tokens), not through
moe_route_topk, so their selections are compared here through the layer's
idx_out / w_out:
  - 2000 single-token GLM-scale calls, fresh activations each, in the launch
    configuration the decode benchmark times (one workspace reused);
  - every batch size 1..8 on router layouts that take the warp-reduction
    selection (ungrouped, small groups, all candidates kept, 32 groups) and
    the rank fallback (ungrouped with more than 256 experts), with and
    without expert top-p.
Indices bit for bit and weights to 2e-6 relative except tokens whose decision
margin is below 1e-6 (validity-checked instead).

The 4096-token prefill (tensor path) is checked on a deliberate sample of about
128 tokens: the tokens on both sides of every 64-token box edge and 192-token
tile edge in the first tiles of the three most loaded experts and at the start
of their last tile, the first and last token of the shared expert's first and
final chunks, the first tokens of the three least loaded experts, the rest
random; y element by element to 2e-3 of max |y_ref|.
"""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import GpuLayer, OracleLayer, flagged, rel_err, routing_is_valid
from test_gpu_layer import TOL

pytestmark = pytest.mark.gpu


def check_routing(r, idx, w, bias, cfg, rtol=2e-6):
    """idx/w of the CUDA path against the oracle's route r; returns the number
    of flagged tokens."""
    fl = flagged(r)
    assert np.array_equal(idx[~fl], r["idx"][~fl])
    assert np.allclose(w[~fl], r["w"][~fl], rtol=rtol, atol=0)
    for t in np.nonzero(fl)[0]:
        if not np.array_equal(idx[t], r["idx"][t]):
            assert routing_is_valid(r["scores"][t], bias, idx[t], cfg), t
    return int(fl.sum())


@pytest.fixture(scope="module")
def glm(lib):
    return GpuLayer(lib, syn.DECODE)


@pytest.fixture(scope="module")
def glm_orc(orc):
    return OracleLayer(orc, syn.DECODE)


def test_decode_2000_single_token_calls(lib, glm, glm_orc):
    cfg = syn.DECODE
    n = 2000
    x = syn.activations(n, cfg.H, 20_000, "cuda")
    idx = torch.empty((n, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((n, cfg.k), dtype=torch.float32, device="cuda")
    y = torch.empty((n, cfg.H), dtype=torch.float32, device="cuda")
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(1, cfg.H, cfg.I, glm.rcfg))
    for i in range(n):
        lib.moe_layer_forward(x[i:i + 1], glm.gate, glm.bias, glm.rcfg, glm.table, glm.shared, 4,
                              y=y[i:i + 1], idx_out=idx[i:i + 1], w_out=w[i:i + 1], ws=ws)
    torch.cuda.synchronize()
    assert ws.flags() == 0
    xb = syn.bf16_bits(x)
    r = glm_orc.route(xb)
    idx_h, w_h = idx.cpu().numpy(), w.cpu().numpy()
    n_flag = check_routing(r, idx_h, w_h, glm_orc.bias, cfg)
    assert n_flag < n // 20, n_flag
    # y of a few calls spread over the run, each with its own routing
    pick = np.array([0, 1, 777, 1500, n - 1])
    ref = glm_orc.layer_y(xb[pick], idx_h[pick], w_h[pick])["y"]
    err = rel_err(y.cpu().numpy()[pick], ref)
    assert err <= TOL, err


LAYOUTS = [  # E, n_group, topk_group, k, topp
    (8, 1, 1, 2, 0.0),
    (12, 3, 2, 4, 0.0),
    (9, 3, 3, 9, 0.0),
    (64, 4, 2, 6, 0.0),
    (64, 4, 2, 6, 0.7),
    (160, 1, 1, 6, 0.0),
    (256, 32, 4, 8, 0.5),
    (320, 1, 1, 8, 0.0),
]


@pytest.mark.parametrize("E,n_group,topk_group,k,topp", LAYOUTS)
def test_small_batch_router_layouts(lib, orc, E, n_group, topk_group, k, topp):
    cfg = syn.LayerConfig(f"layout E{E} g{n_group}/{topk_group} k{k}", H=256, I=128, E=E, k=k,
                          n_group=n_group, topk_group=topk_group, bias_amp=0.1, topp=topp)
    L = GpuLayer(lib, cfg)
    OL = OracleLayer(orc, cfg)
    for T in range(1, 9):
        x = syn.activations(T, cfg.H, 900 + 10 * E + T, "cuda")
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        y = lib.moe_layer_forward(x, L.gate, L.bias, L.rcfg, L.table, L.shared, 4, idx_out=idx, w_out=w)
        torch.cuda.synchronize()
        xb = syn.bf16_bits(x)
        r = OL.route(xb)
        idx_h, w_h = idx.cpu().numpy(), w.cpu().numpy()
        check_routing(r, idx_h, w_h, OL.bias, cfg)
        ref = OL.layer_y(xb, idx_h, w_h)["y"]
        err = rel_err(y.cpu().numpy(), ref)
        assert err <= TOL, (T, err)


def _edge_sample(idx, T, E, k, n_total=128, seed=4096):
    """Token sample on the tile structure of the tensor path, from the layer's
    own routing (the choice of tokens only; expected values are the oracle's)."""
    tokens = {e: np.nonzero((idx == e).any(axis=1))[0] for e in range(E)}
    counts = np.array([len(tokens[e]) for e in range(E)])
    pick = set()
    for e in np.argsort(-counts, kind="stable")[:3]:
        lst = tokens[e]
        assert len(lst) > 192, counts[e]
        # 64-token box edges of the first tile, tile edges, the last tile's start
        edges = {64, 128, 192, 384, 576, (len(lst) - 1) // 192 * 192}
        for edge in sorted(edges):
            if 0 < edge < len(lst):
                pick.update(int(t) for t in lst[edge - 1:edge + 1])
        pick.update([int(lst[0]), int(lst[-1])])
    last0 = (T - 1) // 192 * 192
    pick.update([0, 191, 192, last0, T - 1])
    live = [e for e in range(E) if counts[e] > 0]
    for e in sorted(live, key=lambda e: counts[e])[:3]:
        pick.update(int(t) for t in tokens[e][:4])
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.array(sorted(pick)))
    if len(pick) < n_total:
        pick.update(int(t) for t in rng.choice(rest, n_total - len(pick), replace=False))
    return np.array(sorted(pick)), counts


def test_prefill_tile_edge_sample(lib, glm, orc):
    cfg = syn.PREFILL.with_(bias_kind="zipf")
    OL = OracleLayer(orc, cfg)
    bias = syn.router_bias(cfg, 0, "cuda")
    T = cfg.T
    x = syn.activations(T, cfg.H, 4097, "cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    y = lib.moe_layer_forward(x, glm.gate, bias, glm.rcfg, glm.table, glm.shared, 4, idx_out=idx, w_out=w)
    torch.cuda.synchronize()
    idx_h, w_h = idx.cpu().numpy(), w.cpu().numpy()
    sample, counts = _edge_sample(idx_h, T, cfg.E, cfg.k)
    assert counts.max() > 2 * 192, counts.max()
    xb = syn.bf16_bits(x)[sample]
    r = OL.route(xb)
    check_routing(r, idx_h[sample], w_h[sample], OL.bias, cfg)
    ref = OL.layer_y(xb, idx_h[sample], w_h[sample])["y"]
    got = y.cpu().numpy()[sample]
    scale = np.max(np.abs(ref))
    bad = np.abs(got - ref) > TOL * scale
    assert not bad.any(), (sample[np.nonzero(bad.any(axis=1))[0]], rel_err(got, ref))
