"""The rows that widen the layer, on the GPU against the oracle:
  - a stack of MoE layers chained by RMSNorm and fp32 residual adds
    (moe_stack_forward), the oracle running its own norm, router and layer
    chain from the same starting residual;
  - int8 and int2 experts through moe_layer_forward (decode and AUTO batches);
  - adaptive expert top-p at layer level (dropped slots skip their expert);
  - the MTP-verify shape: a few draft tokens close to one another, so the
    batch union shares most experts.
Indices bit for bit except flagged near-ties (validity-checked instead);
max |y - y_ref| <= 2e-3 max |y_ref| per layer."""
import copy

import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import GpuLayer, OracleLayer, flagged, rel_err, routing_is_valid
from test_gpu_layer import TOL, run_and_check

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# stack: resid_{l+1} = resid_l + MoE_l(bf16(rmsnorm(resid_l)))
# ---------------------------------------------------------------------------
def _bf16_bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def stack_check(lib, orc, cfg, n_layers, T, seed):
    layers = [GpuLayer(lib, cfg, layer=l) for l in range(n_layers)]
    oracle = [OracleLayer(orc, cfg, layer=l) for l in range(n_layers)]
    resid0 = syn.normal((T, cfg.H), 1.0, syn.seed_of("resid", T, cfg.H, seed), "cuda")
    resid = resid0.clone()
    li = torch.empty((n_layers, T, cfg.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((n_layers, T, cfg.k), dtype=torch.int32, device="cuda")
    lib.moe_stack_forward(resid, [(L.gate, L.bias, L.table, L.shared, L.bits) for L in layers],
                          layers[0].rcfg, cfg.I, eps=1e-6, layer_inputs=li, idx_out=idx)
    torch.cuda.synchronize()
    gpu_li = [syn.bf16_bits(li[l]) for l in range(n_layers)]
    gpu_idx = idx.cpu().numpy()

    r = resid0.cpu().numpy().astype(np.float64)
    for l, OL in enumerate(oracle):
        xb, _ = orc.rmsnorm_bf16(r, 1e-6)
        # the layer input: bf16 of the same norm, rounded from fp32 on the GPU
        # and from fp64 in the oracle -> equal up to one bf16 ulp on layer 0.
        # After that the two chains carry different residuals: one ulp flipped
        # by that rounding (0.4% of one input element) moves the layer's output
        # by up to ~1e-4 of max |y| (a single-layer run on identical inputs
        # agrees to 1e-6), so later inputs also get the layer tolerance, scaled
        # by the norm like everything else
        gv, ov = _bf16_bits_to_f64(gpu_li[l]), _bf16_bits_to_f64(xb)
        allow = np.abs(ov) * 2.0 ** -7 + (TOL * l * np.max(np.abs(ov)) if l else 1e-30)
        assert np.all(np.abs(gv - ov) <= allow), (l, float(np.max(np.abs(gv - ov) - allow)))
        ro = OL.route(xb)
        fl = flagged(ro)
        use_idx, use_w = ro["idx"].copy(), ro["w"].copy()
        assert np.array_equal(gpu_idx[l][~fl], ro["idx"][~fl]), l
        for t in np.nonzero(fl)[0]:
            if not np.array_equal(gpu_idx[l][t], ro["idx"][t]):
                assert routing_is_valid(ro["scores"][t], OL.bias, gpu_idx[l][t], cfg)
                use_idx[t] = gpu_idx[l][t]
                sc = ro["scores"][t][np.maximum(use_idx[t], 0)]
                use_w[t] = np.where(use_idx[t] >= 0, sc / sc[use_idx[t] >= 0].sum() * cfg.rsf, 0)
        r = r + OL.layer_y(xb, use_idx, use_w)["y"]
    out = resid.cpu().numpy()
    err = rel_err(out, r)
    assert err <= TOL * n_layers, err
    return err


def test_stack_tiny_three_layers(lib, orc):
    stack_check(lib, orc, syn.TINY, n_layers=3, T=4, seed=11)


@pytest.mark.parametrize("T", [1, 4])
def test_stack_glm_two_layers_decode(lib, orc, T):
    """T = 1 runs the fused router + streaming GEMV kernels, T = 4 the fused
    decode-layer kernel, both two GLM-scale layers deep."""
    stack_check(lib, orc, syn.DECODE, n_layers=2, T=T, seed=12)


# ---------------------------------------------------------------------------
# int8 / int2 experts
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [8, 2])
@pytest.mark.parametrize("T", [1, 4, 64])
def test_layer_tiny_int8_int2(lib, orc, bits, T):
    L = GpuLayer(lib, syn.TINY, bits=bits)
    OL = OracleLayer(orc, syn.TINY, bits=bits)
    run_and_check(lib, L, OL, syn.activations(T, syn.TINY.H, 5000 + T, "cuda"))


@pytest.mark.parametrize("bits", [8, 2])
def test_layer_glm_decode_int8_int2(lib, orc, bits):
    L = GpuLayer(lib, syn.DECODE, bits=bits)
    OL = OracleLayer(orc, syn.DECODE, bits=bits)
    for seed in (1, 2):
        run_and_check(lib, L, OL, syn.activations(1, syn.DECODE.H, 6000 + seed, "cuda"))
    del L
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# adaptive expert top-p and the MTP-verify shape (GLM-scale int4 layer)
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def glm(lib):
    return GpuLayer(lib, syn.DECODE)


def _with_cfg(lib, L, cfg):
    L2 = copy.copy(L)
    L2.cfg = cfg
    L2.rcfg = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
    return L2


@pytest.mark.parametrize("T", [1, 4])
def test_layer_expert_topp(lib, orc, glm, T):
    cfg = syn.DECODE.with_(topp=0.7)
    L = _with_cfg(lib, glm, cfg)
    OL = OracleLayer(orc, cfg)
    x = syn.activations(T, cfg.H, 7000 + T, "cuda")
    idx, _, _ = lib.moe_route_topk(x, L.gate, L.bias, L.rcfg)
    assert (idx < 0).any(), "top-p 0.7 should drop some slots"
    run_and_check(lib, L, OL, x)


@pytest.mark.parametrize("T", [2, 4])
def test_layer_mtp_verify_shape(lib, orc, glm, T):
    """Drafts x_t = x_0 + 0.05 n_t (bf16) under the Zipf-skewed router: most
    experts are shared by the drafts, which the batch union reads once."""
    cfg = syn.SMALL_BATCH.with_(T=T)
    bias = syn.router_bias(cfg, 0, "cuda")
    x0 = syn.normal((1, cfg.H), 1.0, syn.seed_of("mtp-x0", T, cfg.H, 0), "cuda")
    noise = syn.normal((T, cfg.H), 0.05, syn.seed_of("mtp-noise", T, cfg.H, 0), "cuda")
    x = (x0 + noise).to(torch.bfloat16)
    idx, _, _ = lib.moe_route_topk(x, glm.gate, bias, glm.rcfg)
    n_unique = len(np.unique(idx.cpu().numpy()))
    assert n_unique < T * cfg.k
    OL = OracleLayer(orc, cfg)
    run_and_check(lib, glm, OL, x, bias=bias)
