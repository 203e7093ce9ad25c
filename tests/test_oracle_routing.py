"""Pins for the oracle's routing and dispatch (CPU only).

Each check compares the oracle with something other than itself: values
worked by hand from the pages (tests/golden/), brute-force enumeration of
group and expert subsets, invariants that the definitions imply, closed forms,
and library routines (torch's bfloat16 conversion).
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "routing_worked_example.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _route(z, bias, **kw):
    return O.route(np.asarray(z, np.float64), None if bias is None else np.asarray(bias), **kw)


# ---------------------------------------------------------------- number formats

def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, -1.0, 3.0e38, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
                         -(1.0 + 2.0 ** -8), 255.5, 256.5, 257.0]]).astype(np.float32)
    ours = O.round_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_round_f32_known_values():
    # binary32 keeps 24 significant bits: 1 + 2^-23 is the next value after 1;
    # halfway cases go to the even significand
    u = 2.0 ** -23
    cases = [
        (1.0 + u / 2, 1.0),                          # halfway, 1.0 is even
        (1.0 + 3 * u / 2, 1.0 + 2 * u),              # halfway, 1 + 2u is even
        (1.0 + u / 2 + 2.0 ** -40, 1.0 + u),         # just above halfway rounds up
        (1.0 + u / 2 - 2.0 ** -40, 1.0),             # just below rounds down
        (-(1.0 + 3 * u / 2), -(1.0 + 2 * u)),        # symmetric in sign
        (2.0 ** -149, 2.0 ** -149),                  # smallest subnormal is kept
        (2.0 ** -150, 0.0),                          # halfway to 0, 0 is even
        (3 * 2.0 ** -151, 2.0 ** -149),              # 0.75 of the smallest subnormal
        (1.0 / 3.0, 11184811 * 2.0 ** -25),          # nearest binary32 to 1/3
        (float(2 ** 24 + 1), float(2 ** 24)),        # integers past 2^24 lose the last bit
    ]
    v = np.array([c[0] for c in cases])
    np.testing.assert_array_equal(O.round_f32(v), np.array([c[1] for c in cases]))


def test_round_f32_matches_torch():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)
    ref = torch.from_numpy(v).to(torch.float32).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_f32(v), ref)


def test_to_f64_from_bf16_bits():
    v = torch.randn(1000, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    bits = v.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.to_f64(bits), v.to(torch.float64).numpy())


# ---------------------------------------------------------------- hand-worked examples

def _golden_sigmoid(name):
    g = _golden()[name]
    s = np.array(g["s"])
    z = np.log(s / (1 - s))[None, :]
    # with x = z and W_r = identity the logits are z (page "Expert scores": z = x W_r)
    zz = O.router_logits(z, np.eye(len(s)))
    r = _route(zz, g["bias"], n_groups=g["n_groups"], topk_groups=g["topk_groups"],
               topk=g["topk"], score_func=g["score_func"], route_scale=g["route_scale"])
    assert r["groups"][0].tolist() == g["expected_groups"]
    assert r["idx"][0].tolist() == g["expected_idx"]
    np.testing.assert_allclose(r["weights"][0], g["expected_weights"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["margin"][0], g["expected_margin"], rtol=0, atol=1e-12)


def test_golden_sigmoid_groups():
    _golden_sigmoid("sigmoid_groups")


def test_golden_group_gap_decides_margin():
    _golden_sigmoid("sigmoid_group_gap_decides")


def test_golden_softmax():
    g = _golden()["softmax_plain"]
    r = _route(np.array([g["z"]]), None, n_groups=1, topk_groups=1, topk=g["topk"],
               score_func="softmax", route_scale=g["route_scale"])
    assert r["idx"][0].tolist() == g["expected_idx"]
    np.testing.assert_allclose(r["weights"][0], g["expected_weights"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["margin"][0], g["expected_margin"], rtol=0, atol=1e-12)


def test_golden_dispatch():
    g = _golden()["dispatch"]
    d = O.dispatch(np.array(g["idx"]), g["n_experts"])
    assert d["counts"].tolist() == g["expected_counts"]
    assert d["offsets"].tolist() == g["expected_offsets"]
    assert d["src"].tolist() == g["expected_src"]
    assert d["pos"].tolist() == g["expected_pos"]


# ---------------------------------------------------------------- brute force

def _brute_force(z, bias, n_groups, topk_groups, topk, score_func):
    """Independent restatement by enumeration: the kept groups are the unique
    subset whose every member scores above every non-member; the experts are
    the k-subset of the eligible ones with the largest sum of biased scores."""
    E = len(z)
    if score_func == "sigmoid":
        s = [1.0 / (1.0 + math.exp(-v)) for v in z]
    else:
        m = max(z)
        ex = [math.exp(v - m) for v in z]
        s = [v / sum(ex) for v in ex]
    b = [s[e] + (bias[e] if bias is not None else 0.0) for e in range(E)]
    per = E // n_groups
    eligible = list(range(E))
    kept = None
    if n_groups > 1:
        def gscore(gi):
            vals = sorted(b[gi * per:(gi + 1) * per], reverse=True)
            return vals[0] + vals[1] if bias is not None else vals[0]
        gs = [gscore(gi) for gi in range(n_groups)]
        winners = [set(S) for S in itertools.combinations(range(n_groups), topk_groups)
                   if all(gs[i] > gs[o] for i in S for o in range(n_groups) if o not in S)]
        assert len(winners) == 1
        kept = sorted(winners[0])
        eligible = [e for e in range(E) if e // per in winners[0]]
    best, best_sum, second = None, -math.inf, -math.inf
    for S in itertools.combinations(eligible, topk):
        tot = sum(b[e] for e in S)
        if tot > best_sum:
            best, best_sum, second = S, tot, best_sum
        elif tot > second:
            second = tot
    assert best_sum > second  # unique optimum on random inputs
    # the decisive gaps, from the enumerated sets and no sorting: kept groups
    # against dropped ones, chosen experts against eligible ones left out, and
    # the closest pair among the chosen (which fixes their order)
    gaps = []
    if n_groups > 1 and topk_groups < n_groups:
        gaps.append(min(gs[i] for i in kept) - max(gs[o] for o in range(n_groups) if o not in kept))
    rest = [e for e in eligible if e not in best]
    if rest:
        gaps.append(min(b[e] for e in best) - max(b[e] for e in rest))
    gaps += [abs(b[i] - b[j]) for i, j in itertools.combinations(best, 2)]
    margin = min(gaps) if gaps else math.inf
    return kept, set(best), s, b, margin


CASES = [
    # E, G, TG, k, score, bias
    (8, 4, 2, 3, "sigmoid", True),
    (16, 4, 2, 4, "sigmoid", True),
    (16, 8, 3, 5, "sigmoid", True),
    (12, 3, 1, 2, "sigmoid", True),
    (16, 4, 2, 4, "softmax", False),
    (16, 4, 3, 6, "sigmoid", False),
    (10, 1, 1, 3, "softmax", False),
    (10, 1, 1, 4, "sigmoid", True),
    (32, 8, 4, 8, "sigmoid", True),
]


@pytest.mark.parametrize("E,G,TG,k,score,has_bias", CASES)
def test_brute_force_routing(E, G, TG, k, score, has_bias):
    rng = np.random.default_rng(E * 1000 + G * 100 + k)
    T = 12 if E >= 32 else 25
    z = rng.standard_normal((T, E)) * 1.5
    bias = rng.standard_normal(E) * 0.1 if has_bias else None
    r = _route(z, bias, n_groups=G, topk_groups=TG, topk=k, score_func=score, route_scale=1.7)
    for t in range(T):
        kept, chosen, s, b, margin = _brute_force(list(z[t]), None if bias is None else list(bias),
                                                  G, TG, k, score)
        assert math.isclose(r["margin"][t], margin, rel_tol=0, abs_tol=1e-12)
        if G > 1:
            assert r["groups"][t].tolist() == kept
        assert set(r["idx"][t].tolist()) == chosen
        # descending biased score
        bt = [b[e] for e in r["idx"][t]]
        assert all(bt[i] > bt[i + 1] for i in range(k - 1))
        # weights: unbiased scores, renormalised for sigmoid, then scaled
        wt = [s[e] for e in r["idx"][t]]
        if score == "sigmoid":
            wt = [v / sum(wt) for v in wt]
        np.testing.assert_allclose(r["weights"][t], np.array(wt) * 1.7, rtol=1e-12)


@pytest.mark.parametrize("E,G,TG,k,score,has_bias", [c for c in CASES if c[5]])
def test_margin_is_the_routing_decision_radius(E, G, TG, k, score, has_bias):
    """Shifting every biased score by less than margin/4 (a group's top-2 sum
    then moves by less than margin/2) leaves the brute-force routing
    unchanged; pushing the deciding pair towards each other by a little more
    than the margin changes it. The shifts go through the bias, one token at
    a time."""
    rng = np.random.default_rng(100 + E + k)
    T = 10
    z = rng.standard_normal((T, E)) * 1.5
    bias = rng.standard_normal(E) * 0.1
    kw = dict(n_groups=G, topk_groups=TG, topk=k, score_func=score, route_scale=1.0)
    r = _route(z, bias, **kw)
    per = E // G
    for t in range(T):
        m = r["margin"][t]
        ref = _brute_force(list(z[t]), list(bias), G, TG, k, score)
        for _ in range(3):
            d = rng.uniform(-1, 1, E) * 0.249 * m
            got = _brute_force(list(z[t]), list(bias + d), G, TG, k, score)
            assert got[0] == ref[0] and got[1] == ref[1]
            rt = _route(z[t:t + 1], bias + d, **kw)
            assert rt["idx"][0].tolist() == r["idx"][t].tolist()
        # the deciding pair, pushed across its gap
        b = ref[3]
        idx = r["idx"][t].tolist()
        d = np.zeros(E)
        pair_gaps = [(abs(b[i] - b[j]), i, j) for a, i in enumerate(idx) for j in idx[a + 1:]]
        elig = [e for e in range(E) if G == 1 or e // per in set(ref[0])]
        rest = [e for e in elig if e not in idx]
        if rest:
            worst = min(idx, key=lambda e: b[e])
            best_out = max(rest, key=lambda e: b[e])
            pair_gaps.append((b[worst] - b[best_out], worst, best_out))
        gap, hi, lo = min(pair_gaps)
        if gap <= m * (1 + 1e-9):
            d[hi] -= 0.6 * gap
            d[lo] += 0.6 * gap
        else:
            # the group gap decides: lower every member of the worst kept
            # group and raise every member of the best dropped group
            gs = {gi: sorted(b[gi * per:(gi + 1) * per], reverse=True) for gi in range(G)}
            score_g = {gi: v[0] + v[1] for gi, v in gs.items()}
            kg = min(ref[0], key=lambda gi: score_g[gi])
            dg = max((gi for gi in range(G) if gi not in ref[0]), key=lambda gi: score_g[gi])
            d[kg * per:(kg + 1) * per] -= 0.3 * m
            d[dg * per:(dg + 1) * per] += 0.3 * m
        rt = _route(z[t:t + 1], bias + d, **kw)
        flipped = _brute_force(list(z[t]), list(bias + d), G, TG, k, score)
        assert rt["idx"][0].tolist() != r["idx"][t].tolist()
        assert (flipped[0], flipped[1]) != (ref[0], ref[1]) or \
            sorted(idx, key=lambda e: -flipped[3][e]) != idx


def pin_brute_force_margins():
    """Every brute-force shape family in one call (used by the planted-mistake
    tests, which call pins without arguments)."""
    for case in CASES:
        test_brute_force_routing(*case)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("E,G,TG,k,score,has_bias", CASES)
def test_routing_invariants(E, G, TG, k, score, has_bias):
    rng = np.random.default_rng(7 + E + k)
    T = 300
    z = rng.standard_normal((T, E))
    bias = rng.standard_normal(E) * 0.1 if has_bias else None
    r = _route(z, bias, n_groups=G, topk_groups=TG, topk=k, score_func=score, route_scale=2.5)
    idx, w = r["idx"], r["weights"]
    assert idx.shape == (T, k)
    assert all(len(set(row)) == k for row in idx.tolist())
    assert idx.min() >= 0 and idx.max() < E
    if score == "sigmoid":
        np.testing.assert_allclose(w.sum(-1), 2.5, rtol=0, atol=1e-12)
    else:
        assert np.all(w.sum(-1) <= 2.5 + 1e-12)
    assert np.all(w > 0)
    if G > 1:
        per = E // G
        for t in range(T):
            assert set((idx[t] // per).tolist()) <= set(r["groups"][t].tolist())
    assert np.all(r["margin"] > 0)


def test_dispatch_invariants():
    rng = np.random.default_rng(3)
    T, k, E = 500, 6, 40
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    d = O.dispatch(idx, E)
    assert d["counts"].sum() == T * k
    np.testing.assert_array_equal(d["counts"], [np.sum(idx == e) for e in range(E)])
    np.testing.assert_array_equal(d["offsets"][1:] - d["offsets"][:-1], d["counts"])
    assert d["offsets"][0] == 0
    pos = d["pos"].reshape(-1)
    assert sorted(pos.tolist()) == list(range(T * k))           # bijection
    for t in range(T):
        for j in range(k):
            p = d["pos"][t, j]
            e = idx[t, j]
            assert d["src"][p] == t
            assert d["offsets"][e] <= p < d["offsets"][e + 1]
    for e in range(E):                                          # ascending tokens
        seg = d["src"][d["offsets"][e]:d["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)


# ---------------------------------------------------------------- closed forms

def test_zero_router_sigmoid_selects_by_bias():
    # W_r = 0: every score is exactly 0.5, selection is by the bias alone,
    # and each weight is route_scale / k exactly.
    E, G, TG, k, T = 16, 4, 2, 4, 10
    bias = np.zeros(E)
    # group 1 (experts 4..7) and group 3 (12..15) get the two largest top-2 sums
    bias[[5, 6]] = [0.30, 0.20]          # group 1: top-2 sum 1.5
    bias[[12, 15]] = [0.25, 0.10]        # group 3: top-2 sum 1.35
    bias[0] = 0.28                       # group 0: top-2 sum 1.28 (only one high)
    x = np.random.default_rng(0).standard_normal((T, 32))
    z = O.router_logits(x, np.zeros((E, 32)))
    r = O.route(z, bias, n_groups=G, topk_groups=TG, topk=k, score_func="sigmoid", route_scale=2.5)
    for t in range(T):
        assert r["groups"][t].tolist() == [1, 3]
        assert r["idx"][t].tolist() == [5, 12, 6, 15]
    np.testing.assert_array_equal(r["weights"], np.full((T, k), 2.5 / k))
    d = O.dispatch(r["idx"], E)
    assert d["counts"].tolist() == [T if e in (5, 6, 12, 15) else 0 for e in range(E)]


def test_zero_router_softmax_ties_to_lowest_index():
    E, k, T = 64, 6, 5
    z = O.router_logits(np.ones((T, 8)), np.zeros((E, 8)))
    r = O.route(z, None, n_groups=1, topk_groups=1, topk=k, score_func="softmax", route_scale=1.0)
    for t in range(T):
        assert r["idx"][t].tolist() == list(range(k))
    np.testing.assert_allclose(r["weights"], 1.0 / E, rtol=1e-15)


def test_one_hot_bias_always_chosen():
    rng = np.random.default_rng(5)
    E, G, TG, k, T = 32, 8, 4, 8, 200
    bias = np.zeros(E)
    bias[19] = 10.0
    z = rng.standard_normal((T, E)) * 3
    r = O.route(z, bias, n_groups=G, topk_groups=TG, topk=k, score_func="sigmoid", route_scale=1.0)
    assert np.all(r["idx"][:, 0] == 19)
    assert np.all(np.any(r["groups"] == 19 // 4, axis=1))
