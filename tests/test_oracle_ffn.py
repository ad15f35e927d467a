"""Pins for the oracle's SwiGLU expert FFN and the MoE layer combination."""
from fractions import Fraction
import math

import numpy as np
import pytest


def _qexpert(orc, wg, wu, wd, bits=4):
    qg, sg = orc.quantize_rows(wg, bits)
    qu, su = orc.quantize_rows(wu, bits)
    qd, sd = orc.quantize_rows(wd, bits)
    return orc.Expert(qg, sg, qu, su, qd, sd, bits)


def test_identity_like_expert_closed_form(orc):
    """W_g = c_g [I | 0], W_u = c_u [I | 0], W_d = c_d [I ; 0] with c = 7 * 2^-m,
    so every row max is c, scale = c / 7 = 2^-m exactly and the diagonal code is 7:
    dequantisation is exact and y_j = c_d * silu(c_g x_j) * c_u x_j for j < I,
    0 for j >= I (tiny workload sizes H = 256, I = 128)."""
    H, I = 256, 128
    cg, cu, cd = 7 * 2.0 ** -3, 7 * 2.0 ** -2, 7 * 2.0 ** -4
    eye = np.eye(I, H, dtype=np.float32)
    ex = _qexpert(orc, cg * eye, cu * eye, cd * np.eye(H, I, dtype=np.float32))
    rng = np.random.default_rng(11)
    xb = orc.f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32))
    x = orc.bf16_bits_to_f64(xb)
    y = orc.expert_ffn(xb, ex, H, I)
    g = cg * x[:, :I]
    want = np.zeros((3, H))
    want[:, :I] = cd * (g / (1.0 + np.exp(-g))) * (cu * x[:, :I])
    assert np.allclose(y, want, rtol=1e-14, atol=1e-300)
    assert np.all(y[:, I:] == 0)


def test_zero_up_projection_gives_zero(orc):
    rng = np.random.default_rng(12)
    H, I = 64, 32
    ex = _qexpert(orc, (rng.standard_normal((I, H)) * 0.02).astype(np.float32),
                  np.zeros((I, H), np.float32),
                  (rng.standard_normal((H, I)) * 0.02).astype(np.float32))
    xb = orc.f32_to_bf16_bits(rng.standard_normal((2, H)).astype(np.float32))
    assert np.all(orc.expert_ffn(xb, ex, H, I) == 0)


def test_ffn_matches_exact_rational_evaluation(orc):
    """Brute force on a tiny expert: every product and sum in exact rationals
    (only silu's exp in fp64), from the unpacked codes and scales; the fp64 oracle
    must agree to within the fp64 rounding bound of its sums."""
    rng = np.random.default_rng(13)
    H, I = 32, 16
    wg = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    wu = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    wd = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    ex = _qexpert(orc, wg, wu, wd)
    xb = orc.f32_to_bf16_bits(rng.standard_normal((2, H)).astype(np.float32))
    x = orc.bf16_bits_to_f64(xb)
    cg, cu, cd = (orc.unpack(q, c, 4) for q, c in ((ex.qg, H), (ex.qu, H), (ex.qd, I)))
    y = orc.expert_ffn(xb, ex, H, I)
    for t in range(2):
        xf = [Fraction(float(v)) for v in x[t]]
        h = []
        for i in range(I):
            g = sum(Fraction(int(cg[i, j])) * Fraction(float(ex.sg[i])) * xf[j] for j in range(H))
            u = sum(Fraction(int(cu[i, j])) * Fraction(float(ex.su[i])) * xf[j] for j in range(H))
            gf = float(g)
            h.append(Fraction(gf / (1.0 + math.exp(-gf))) * u)
        for j in range(H):
            exact = sum(Fraction(int(cd[j, i])) * Fraction(float(ex.sd[j])) * h[i]
                        for i in range(I))
            bound = 1e-13 * float(sum(abs(Fraction(int(cd[j, i])) * Fraction(float(ex.sd[j])) * h[i])
                                      for i in range(I))) + 1e-300
            assert abs(y[t, j] - float(exact)) <= bound


def test_expert_rows_are_not_transposed(orc):
    """H != I, and a one-hot gate/up row picks one input column: catches a
    transposed or mis-strided operand."""
    H, I = 64, 32
    wg = np.zeros((I, H), np.float32)
    wu = np.zeros((I, H), np.float32)
    wd = np.zeros((H, I), np.float32)
    wg[5, 40] = 0.875
    wu[5, 40] = 1.75
    wd[60, 5] = 0.4375
    ex = _qexpert(orc, wg, wu, wd)
    xb = orc.f32_to_bf16_bits(np.linspace(-2, 2, H, dtype=np.float32)[None, :])
    x = orc.bf16_bits_to_f64(xb)[0]
    y = orc.expert_ffn(xb, ex, H, I)[0]
    g = 0.875 * x[40]
    assert y[60] == pytest.approx(0.4375 * g / (1 + math.exp(-g)) * 1.75 * x[40], rel=1e-14)
    assert np.count_nonzero(y) == 1


def _random_layer(orc, rng, H, I, E, bits=4):
    experts = []
    for _ in range(E):
        experts.append(_qexpert(orc, *(
            (rng.standard_normal(s) * 0.02).astype(np.float32)
            for s in ((I, H), (I, H), (H, I))), bits=bits))
    shared = _qexpert(orc, *((rng.standard_normal(s) * 0.02).astype(np.float32)
                             for s in ((I, H), (I, H), (H, I))), bits=bits)
    G = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    return experts, shared, G, bias


@pytest.mark.parametrize("bits", [4, 8, 2])
def test_layer_is_weighted_sum_of_experts_plus_shared(orc, bits):
    rng = np.random.default_rng(14 + bits)
    H, I, E, k = 64, 32, 8, 2
    experts, shared, G, bias = _random_layer(orc, rng, H, I, E, bits)
    xb = orc.f32_to_bf16_bits(rng.standard_normal((5, H)).astype(np.float32))
    out = orc.layer(xb, G, bias, experts, shared, H, I, k, rsf=2.5)
    r = orc.route(xb, G, bias, k, rsf=2.5)
    assert np.array_equal(out["idx"], r["idx"]) and np.array_equal(out["w"], r["w"])
    for t in range(5):
        want = orc.expert_ffn(xb[t:t + 1], shared, H, I)[0].copy()
        for i in range(k):
            want += float(r["w"][t, i]) * orc.expert_ffn(xb[t:t + 1], experts[r["idx"][t, i]],
                                                         H, I)[0]
        assert np.allclose(out["y"][t], want, rtol=1e-13, atol=1e-15)


def test_layer_teacher_forced_routing_and_missing_expert(orc):
    rng = np.random.default_rng(15)
    H, I, E, k = 64, 32, 4, 2
    experts, shared, G, bias = _random_layer(orc, rng, H, I, E)
    xb = orc.f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32))
    idx = np.array([[3, 1], [0, 2], [1, 3]], np.int32)
    w = np.array([[0.5, 0.25], [1.0, 2.0], [0.125, 0.0]], np.float32)
    out = orc.layer(xb, G, bias, experts, None, H, I, k, idx_in=idx, w_in=w)
    want = np.zeros((3, H))
    for t in range(3):
        for i in range(k):
            want[t] += float(w[t, i]) * orc.expert_ffn(xb[t:t + 1], experts[idx[t, i]], H, I)[0]
    assert np.allclose(out["y"], want, rtol=1e-13, atol=1e-15)
    sparse = [experts[0], None, experts[2], None]
    with pytest.raises(orc.OracleError):
        orc.layer(xb, G, bias, sparse, None, H, I, k, idx_in=idx, w_in=w)


def test_rmsnorm_closed_form(orc):
    v = np.full((2, 16), 3.0)
    v[1] = -0.5
    bits, f = orc.rmsnorm_bf16(v, eps=1e-6)
    assert np.allclose(f[0], 3.0 / math.sqrt(9.0 + 1e-6), rtol=1e-15)
    assert np.allclose(f[1], -0.5 / math.sqrt(0.25 + 1e-6), rtol=1e-15)
    assert np.array_equal(bits, orc.double_to_bf16_bits(f))
    z, fz = orc.rmsnorm_bf16(np.zeros((1, 8)))
    assert np.all(fz == 0)
