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


# Sigmoid closed forms.  For r > 0, sigmoid(ln r) = r / (1 + r).  The logits below
# are exact fp32 values (fp32(ln r), or 0, or 20) and the fp32 rounding of the
# true sigmoid of each is the rational r/(1+r) (resp. 1/2, 1): the distance of
# sigmoid(fp32(ln r)) from r/(1+r) is at most 0.11 ulp of the result below the
# rounding boundary, derived from |fp32(ln r) - ln r| <= 2^-24 * |ln r| and
# sigmoid' = s(1 - s).  sigmoid(20) = 1 - 2.06e-9 lies within 2^-25 of 1.
SIGMOID_PINS = [
    ("0x0p+0", 0.5),
    ("0x1.193ea8p+0", 0.75),     # fp32(ln 3)
    ("-0x1.193ea8p+0", 0.25),    # fp32(-ln 3)
    ("0x1.f2272ap+0", 0.875),    # fp32(ln 7)
    ("-0x1.f2272ap+0", 0.125),   # fp32(-ln 7)
    ("0x1.5aa164p+1", 0.9375),   # fp32(ln 15)
    ("0x1.4p+4", 1.0),           # 20
]


def test_scores_closed_form_sigmoid(orc):
    """Token scores against closed forms, with the logit formed three ways so
    that a transposed gate matrix, a dropped product or a wrong operand shows:
    token 0 is one-hot 1.0 at column 3 (logit = G[e,3]); token 1 is 2.0 at column
    10 with G[e,10] = logit/2; token 2 is 1.0 at column 20 and 2.0 at column 41
    with G[e,20] = logit/2 and G[e,41] = logit/4 (all exact in fp32)."""
    E, H = len(SIGMOID_PINS), 64
    t_of = np.array([float.fromhex(h) for h, _ in SIGMOID_PINS], np.float32)
    want = np.array([v for _, v in SIGMOID_PINS], np.float32)
    G = np.zeros((E, H), np.float32)
    G[:, 3] = t_of
    G[:, 10] = t_of / np.float32(2)
    G[:, 20] = t_of / np.float32(2)
    G[:, 41] = t_of / np.float32(4)
    x = np.zeros((3, H), np.float32)
    x[0, 3] = 1.0
    x[1, 10] = 2.0
    x[2, 20] = 1.0
    x[2, 41] = 2.0
    xb = orc.f32_to_bf16_bits(x)
    # the rows of G other than those columns are zero, so every expert's logit is t_of[e]
    r = orc.route(xb, G, np.zeros(E, np.float32), k=1)
    for t in range(3):
        assert np.array_equal(r["scores"][t], want), (t, r["scores"][t], want)
    # one row of G per expert: moving expert e's pin to another row moves its score
    r2 = orc.route(xb, G[::-1].copy(), np.zeros(E, np.float32), k=1)
    assert np.array_equal(r2["scores"][0], want[::-1])


def test_expert_topp_properties(orc):
    """Expert top-p (the reading of the "--topp" option in "Show HN: running GLM
    5.2 on a slow computer", option list and community benchmarks): on random
    weight vectors the kept slots are the shortest prefix of the slots ranked by
    weight (ties to the lower slot) whose fp32 running sum reaches topp * total;
    kept slots keep their expert and weight (no renormalisation); dropped slots
    read index -1 and weight 0."""
    rng = np.random.default_rng(11)
    n, E = 600, 16
    for k in (2, 5, 8):
        s = rng.uniform(0.01, 0.99, (n, E)).astype(np.float32)
        s[::5] = np.round(s[::5] * 4) / 4  # coarse scores: equal weights
        bias = np.zeros(E, np.float32)
        full = orc.route_from_scores(s, bias, k, 1, 1, 2.5)
        for topp in (0.1, 0.3, 0.5, 0.7, 0.9, 0.99):
            r = orc.route_from_scores(s, bias, k, 1, 1, 2.5, topp=topp)
            for t in range(n):
                w, idx = full["w"][t], full["idx"][t]
                kept = r["idx"][t] >= 0
                m = int(kept.sum())
                assert m >= 1
                assert np.array_equal(r["idx"][t][kept], idx[kept])
                assert np.array_equal(r["w"][t][kept], w[kept])
                assert np.all(r["idx"][t][~kept] == -1) and np.all(r["w"][t][~kept] == 0)
                order = sorted(range(k), key=lambda i: (-float(w[i]), i))
                assert set(np.nonzero(kept)[0].tolist()) == set(order[:m]), (t, topp, w)
                total = np.float32(0)
                for i in range(k):
                    total = np.float32(total + w[i])
                target = np.float32(np.float32(topp) * total)
                run = np.float32(0)
                runs = []
                for i in order:
                    run = np.float32(run + w[i])
                    runs.append(run)
                assert runs[m - 1] >= target
                assert m == 1 or runs[m - 2] < target
