"""Pins for the oracle's router: brute force on tiny inputs, textbook special
cases, the weight-sum invariant, permutation equivariance and the fp32 score
definition."""
import itertools

import numpy as np
import pytest

from golden_io import rows


def brute_force_route(s, bias, k, n_group, topk_group, rsf):
    """Enumerate every set of topk_group groups and every k-subset of their
    experts; keep the set with the largest total (ties: lexicographically
    smallest indices), then order it by descending b (ties: lower index)."""
    E = len(s)
    b = (s.astype(np.float32) + bias.astype(np.float32)).astype(np.float32)
    gs = E // n_group
    if n_group == 1:
        gscore = [0.0]
    else:
        gscore = []
        for g in range(n_group):
            top = sorted(b[g * gs:(g + 1) * gs].tolist(), reverse=True)
            gscore.append(float(np.float32(top[0]) + np.float32(top[1])))
    best_groups = None
    for combo in itertools.combinations(range(n_group), topk_group):
        tot = sum(gscore[g] for g in combo)
        if best_groups is None or tot > best_groups[0]:
            best_groups = (tot, combo)
    cand = [e for e in range(E) if e // gs in best_groups[1]]
    best = None
    for combo in itertools.combinations(cand, k):
        tot = sum(float(b[e]) for e in combo)
        if best is None or tot > best[0]:
            best = (tot, combo)
    chosen = sorted(best[1], key=lambda e: (-float(b[e]), e))
    ssum = np.float32(0)
    for e in chosen:
        ssum = np.float32(ssum + s[e])
    w = [np.float32(np.float32(s[e] / ssum) * np.float32(rsf)) for e in chosen]
    return np.array(chosen, np.int32), np.array(w, np.float32)


def _tiny_cfgs():
    out = []
    for E in (4, 6, 8, 9, 12):
        for n_group in (1, 2, 3):
            if E % n_group or (n_group > 1 and E // n_group < 2):
                continue
            gs = E // n_group
            for tkg in range(1, n_group + 1):
                for k in (1, 2, 3, min(4, tkg * gs)):
                    if k <= tkg * gs:
                        out.append((E, n_group, tkg, k))
    return sorted(set(out))


@pytest.mark.parametrize("E,n_group,topk_group,k", _tiny_cfgs())
def test_router_matches_brute_force(orc, E, n_group, topk_group, k):
    rng = np.random.default_rng(E * 1000 + n_group * 100 + topk_group * 10 + k)
    T = 40
    s = rng.uniform(0.01, 0.99, (T, E)).astype(np.float32)
    s[::4] = np.round(s[::4] * 8) / 8  # coarse values force exact ties
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    if k % 2:
        bias[:] = 0
    r = orc.route_from_scores(s, bias, k, n_group, topk_group, rsf=2.5)
    for t in range(T):
        idx, w = brute_force_route(s[t], bias, k, n_group, topk_group, 2.5)
        assert r["idx"][t].tolist() == idx.tolist(), (t, s[t], bias)
        assert np.array_equal(r["w"][t], w)


def test_n_group_1_zero_bias_is_textbook_topk(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    xb = orc.f32_to_bf16_bits(x)
    G = (rng.standard_normal((10, 64)) * 0.3).astype(np.float32)
    r = orc.route(xb, G, np.zeros(10, np.float32), k=3)
    for t in range(16):
        order = np.argsort(-r["scores"][t].astype(np.float64), kind="stable")[:3]
        assert r["idx"][t].tolist() == order.tolist()


def test_scores_are_fp32_sigmoid_of_exact_logits(orc):
    rng = np.random.default_rng(4)
    T, H, E = 8, 256, 16
    xb = orc.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    G = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    r = orc.route(xb, G, np.zeros(E, np.float32), k=2)
    x = orc.bf16_bits_to_f64(xb)
    logit = (x @ G.astype(np.float64).T).astype(np.float32)  # exact products, fp64 sum
    want = (1.0 / (1.0 + np.exp(-logit.astype(np.float64)))).astype(np.float32)
    assert np.array_equal(r["scores"], want)


def test_weights_sum_to_scaling_factor(orc):
    rng = np.random.default_rng(5)
    T, H, E = 64, 128, 32
    xb = orc.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    G = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
    bias = rng.uniform(-0.05, 0.05, E).astype(np.float32)
    for rsf in (1.0, 2.5):
        r = orc.route(xb, G, bias, k=8, n_group=4, topk_group=2, rsf=rsf)
        tot = r["w"].astype(np.float64).sum(axis=1)
        assert np.all(np.abs(tot - rsf) <= 4 * np.spacing(np.float32(rsf)))
        assert np.all(r["w"] > 0)


def test_k_equals_E_gives_normalised_sigmoid(orc):
    rng = np.random.default_rng(6)
    s = rng.uniform(0.05, 0.95, (10, 6)).astype(np.float32)
    r = orc.route_from_scores(s, np.zeros(6, np.float32), k=6, rsf=1.0)
    for t in range(10):
        w_by_e = np.zeros(6)
        w_by_e[r["idx"][t]] = r["w"][t]
        assert np.allclose(w_by_e, s[t] / s[t].astype(np.float64).sum(), rtol=1e-6)


def test_router_permutation_equivariance(orc):
    rng = np.random.default_rng(8)
    E, n_group = 12, 3
    gs = E // n_group
    s = rng.uniform(0.01, 0.99, (30, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    gperm = np.array([2, 0, 1])
    perm = np.concatenate([gperm[g] * gs + rng.permutation(gs) for g in range(n_group)])
    # new expert perm[e] carries old expert e
    s2 = np.empty_like(s)
    b2 = np.empty_like(bias)
    s2[:, perm] = s
    b2[perm] = bias
    r1 = orc.route_from_scores(s, bias, 4, n_group, 2, 2.5)
    r2 = orc.route_from_scores(s2, b2, 4, n_group, 2, 2.5)
    assert np.array_equal(perm[r1["idx"]], r2["idx"])
    assert np.array_equal(r1["w"], r2["w"])


def test_gaps_are_decision_margins(orc):
    rng = np.random.default_rng(9)
    s = rng.uniform(0.01, 0.99, (50, 16)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, 16).astype(np.float32)
    r = orc.route_from_scores(s, bias, 3, 4, 2, 1.0)
    b = s + bias
    for t in range(50):
        cand = [e for e in range(16) if r["group_sel"][t][e // 4]]
        rest = sorted((float(b[t, e]) for e in cand if e not in r["idx"][t]), reverse=True)
        assert r["gap"][t] == pytest.approx(float(b[t, r["idx"][t][-1]]) - rest[0], abs=0)
        assert r["gap"][t] >= 0 and r["ggap"][t] >= 0


def test_expert_topp_golden(orc):
    for cfg, svals, bvals, topp, want in rows("expert_topp.txt"):
        E, k = (int(v) for v in cfg.split())
        s = np.array([[float(v) for v in svals.split()]], np.float32)
        bias = np.array([float(v) for v in bvals.split()], np.float32)
        r = orc.route_from_scores(s, bias, k, 1, 1, 1.0, topp=float(topp))
        assert r["idx"][0].tolist() == [int(v) for v in want.split()], (cfg, topp)
        kept = r["idx"][0] >= 0
        assert np.all(r["w"][0][~kept] == 0)


def test_bad_router_configs_rejected(orc):
    s = np.full((1, 8), 0.5, np.float32)
    z = np.zeros(8, np.float32)
    for k, ng, tkg in [(9, 1, 1), (2, 3, 1), (5, 4, 2), (1, 8, 1), (2, 2, 3)]:
        with pytest.raises(orc.OracleError):
            orc.route_from_scores(s, z, k, ng, tkg)
