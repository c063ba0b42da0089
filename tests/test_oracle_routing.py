"""Pins of the oracle's routing (sigmoid scores, biased top-k, renormalised weights).

Each check ties the oracle to something other than its own code: brute-force
enumeration of every k-subset, closed forms (sum of weights, ratios of
weights, the zero-router tie), exact integer arithmetic, and hand-derived
worked examples stored under tests/golden/.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _ulp(x):
    return np.spacing(np.abs(np.asarray(x, F32)))


def _brute_topk(keys_row, k):
    """Enumerate every k-subset; keep the one whose members all precede every
    non-member under (key descending, index ascending)."""
    E = len(keys_row)

    def before(a, b):
        return keys_row[a] > keys_row[b] or (keys_row[a] == keys_row[b] and a < b)

    winners = []
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(before(a, b) for a in sub for b in rest):
            winners.append(sub)
    assert len(winners) == 1
    chosen = list(winners[0])
    # order inside the subset by the same total order (insertion sort)
    ordered = []
    for e in chosen:
        pos = 0
        while pos < len(ordered) and before(ordered[pos], e):
            pos += 1
        ordered.insert(pos, e)
    return ordered


@pytest.mark.parametrize("E,k", [(8, 2), (8, 3), (6, 6), (7, 1), (8, 5)])
def test_topk_matches_brute_force(E, k):
    rng = np.random.default_rng(1000 + 10 * E + k)
    for trial in range(60):
        if trial % 3 == 0:
            # coarse grid: many exact ties
            keys = (rng.integers(-3, 4, size=(1, E)) / 4.0).astype(F32)
        else:
            keys = rng.standard_normal((1, E)).astype(F32)
        got = orc.select_topk(keys, k)[0].tolist()
        assert got == _brute_topk(keys[0].tolist(), k)


def test_weights_sum_to_scale_and_follow_score_ratios():
    rng = np.random.default_rng(7)
    T, E, k, scale = 200, 64, 8, 2.5
    logits = rng.standard_normal((T, E)).astype(F32) * F32(1.5)
    bias = (rng.standard_normal(E) * 0.1).astype(F32)
    s = orc.sigmoid_scores(logits)
    idx, w = orc.route(logits, bias, k, scale)
    tot = w.astype(np.float64).sum(axis=1)
    assert np.all(np.abs(tot - scale) <= 4 * k * np.spacing(F32(scale)))
    s_sel = np.take_along_axis(s, idx.astype(np.int64), axis=1).astype(np.float64)
    ratio_w = w[:, 1:].astype(np.float64) / w[:, :1]
    ratio_s = s_sel[:, 1:] / s_sel[:, :1]
    assert np.allclose(ratio_w, ratio_s, rtol=4e-7, atol=0)


def test_bias_changes_selection_not_weights():
    # scores on a 2**-12 grid and biases on a 2**-10 grid keep every key exact,
    # so adding a constant to all biases shifts every key exactly.
    rng = np.random.default_rng(11)
    T, E, k, scale = 64, 32, 4, 2.5
    s = (rng.integers(1, 4096, size=(T, E)) / 4096.0).astype(F32)
    bias = (rng.integers(-200, 200, size=E) / 1024.0).astype(F32)
    idx0 = orc.select_topk(orc.selection_keys(s, bias), k)
    idx1 = orc.select_topk(orc.selection_keys(s, bias + F32(0.25)), k)
    assert np.array_equal(idx0, idx1)
    w0 = orc.routing_weights(s, idx0, scale)
    w1 = orc.routing_weights(s, idx1, scale)
    assert np.array_equal(w0, w1)
    # A bias that forces expert 5 into every selection: the weights of the
    # other selected experts keep their mutual ratios (un-biased scores only).
    b2 = bias.copy()
    b2[5] = F32(4.0)
    idx2 = orc.select_topk(orc.selection_keys(s, b2), k)
    assert np.all(idx2[:, 0] == 5)
    w2 = orc.routing_weights(s, idx2, scale)
    s_sel = np.take_along_axis(s, idx2.astype(np.int64), axis=1).astype(np.float64)
    assert np.allclose(w2 / w2[:, :1], s_sel / s_sel[:, :1], rtol=4e-7)
    # and weights do not depend on the bias value once the set is fixed
    b3 = b2.copy()
    b3[5] = F32(8.0)
    assert np.array_equal(orc.select_topk(orc.selection_keys(s, b3), k), idx2)
    assert np.array_equal(orc.routing_weights(s, idx2, scale), w2)


@pytest.mark.parametrize("k", [1, 2, 3, 8])
def test_zero_router_ties_to_lowest_indices(k):
    T, D, E, scale = 5, 16, 12, 2.5
    h = np.ones((T, D), F32)
    Wr = np.zeros((E, D), F32)
    logits = orc.router_logits(h, Wr)
    s = orc.sigmoid_scores(logits)
    assert np.all(s == F32(0.5))
    idx, w = orc.route(logits, np.zeros(E, F32), k, scale)
    assert np.array_equal(idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(np.abs(w.astype(np.float64) - scale / k) <= 2 * _ulp(scale / k))
    # with a bias, the selection is the top-k of the bias; weights still scale/k
    bias = np.array([0.1, -0.2, 0.3, 0.3, 0.0, -0.05, 0.2, 0.05, -0.3, 0.25, 0.15, 0.0], F32)
    idx, w = orc.route(logits, bias, k, scale)
    expect = sorted(range(E), key=lambda e: (-float(bias[e]), e))[:k]
    assert np.array_equal(idx, np.tile(np.array(expect, np.int32), (T, 1)))
    assert np.all(np.abs(w.astype(np.float64) - scale / k) <= 2 * _ulp(scale / k))


def test_k_equals_E_selects_everything_in_key_order():
    rng = np.random.default_rng(3)
    T, E = 16, 8
    logits = rng.standard_normal((T, E)).astype(F32)
    bias = (rng.standard_normal(E) * 0.1).astype(F32)
    idx, w = orc.route(logits, bias, E, 1.0)
    s = orc.sigmoid_scores(logits)
    keys = orc.selection_keys(s, bias)
    for t in range(T):
        assert sorted(idx[t].tolist()) == list(range(E))
        assert all(keys[t, idx[t, j]] >= keys[t, idx[t, j + 1]] for j in range(E - 1))
        expect = s[t].astype(np.float64) / s[t].astype(np.float64).sum()
        assert np.allclose(w[t].astype(np.float64), expect[idx[t]], rtol=2e-6)


def test_k1_weight_is_exactly_scale():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 16)).astype(F32)
    idx, w = orc.route(logits, np.zeros(16, F32), 1, 2.5)
    assert np.all(w == F32(2.5))
    assert np.array_equal(idx[:, 0], np.argmax(orc.sigmoid_scores(logits), axis=1))


def test_sigmoid_closed_forms():
    ln3 = F32(math.log(3.0))
    s = orc.sigmoid_scores(np.array([[0.0, ln3, -ln3, 40.0, -20.0]], F32))[0]
    assert s[0] == F32(0.5) and s[1] == F32(0.75) and s[2] == F32(0.25)
    assert s[3] == F32(1.0)
    assert abs(float(s[4]) - 2.0611536e-9) < 1e-15
    x = np.linspace(-12, 12, 2001).astype(F32)[None, :]
    a = orc.sigmoid_scores(x)[0].astype(np.float64)
    b = orc.sigmoid_scores(-x)[0].astype(np.float64)
    assert np.all(np.diff(a) >= 0)                  # monotone
    assert np.max(np.abs(a + b - 1.0)) < 1.2e-7     # symmetry s(-x) = 1 - s(x)


def test_router_logits_exact_on_integer_grid():
    # h on a 1/4 grid (bf16-exact), Wr on a 1/16 grid: every partial sum is a
    # multiple of 1/64 below 2**10, so the exact result is representable.
    rng = np.random.default_rng(9)
    T, D, E = 6, 128, 10
    hi = rng.integers(-3, 4, size=(T, D))
    wi = rng.integers(-7, 8, size=(E, D))
    h = (hi / 4.0).astype(F32)
    Wr = (wi / 16.0).astype(F32)
    exact = (hi @ wi.T) / 64.0
    assert np.array_equal(orc.router_logits(h, Wr).astype(np.float64), exact)


def test_nonfinite_logits_rejected():
    with pytest.raises(ValueError):
        orc.sigmoid_scores(np.array([[0.0, np.nan]], F32))


def test_worked_examples():
    with open(os.path.join(GOLDEN, "route_worked_examples.json")) as f:
        g = json.load(f)
    ln3 = np.array([int(g["ln3_fp32"], 16)], np.uint32).view(F32)[0]
    table = {"0": F32(0.0), "ln3": ln3, "-ln3": -ln3}
    for case in g["cases"]:
        logits = np.array([[table[v] for v in case["logits"]]], F32)
        bias = np.array(case["bias"], F32)
        idx, w = orc.route(logits, bias, case["k"], case["scale"])
        assert idx[0].tolist() == case["idx"], case["name"]
        expect = np.array(case["w"])
        assert np.all(np.abs(w[0] - expect) <= 2 * _ulp(expect)), case["name"]


def test_routing_alternatives_cover_near_ties():
    # keys: expert 1 and 3 tie to within 2e-7 at the boundary of a top-2
    ln3 = F32(math.log(3.0))
    logits = np.array([ln3, 0.0, -ln3, 0.0], F32)
    bias = np.array([0.0, 0.0, 0.0, 2e-7], F32)
    cands = orc.routing_alternatives(logits, bias, 2, 2.5, delta=1e-5)
    sets = [sorted(c[0].tolist()) for c in cands]
    assert sets[0] == [0, 3]                      # the strict selection first
    assert sorted(sets) == [[0, 1], [0, 3]]
    for idx, w in cands:
        assert abs(float(w.astype(np.float64).sum()) - 2.5) < 1e-6
    # far from any tie there is exactly one candidate, equal to route()
    rng = np.random.default_rng(12)
    for _ in range(20):
        lg = rng.standard_normal(16).astype(F32)
        b = (rng.standard_normal(16) * 0.1).astype(F32)
        c = orc.routing_alternatives(lg, b, 4, 2.5, delta=0.0)
        idx, w = orc.route(lg[None, :], b, 4, 2.5)
        assert len(c) == 1 and np.array_equal(c[0][0], idx[0]) and np.array_equal(c[0][1], w[0])


# ---------------------------------------------------------------------------
# group-limited routing
# ---------------------------------------------------------------------------
def _brute_grouped(keys_row, k, n_group, topk_group):
    """Every choice of topk_group groups, ranked by the group scores computed
    with sorted() on Python floats; the experts by brute-force top-k inside."""
    E = len(keys_row)
    G = E // n_group
    scores = []
    for g in range(n_group):
        ks = sorted((float(v) for v in keys_row[g * G:(g + 1) * G]), reverse=True)
        scores.append(float(F32(ks[0]) + F32(ks[1])) if G > 1 else ks[0])
    groups = sorted(range(n_group), key=lambda g: (-scores[g], g))[:topk_group]
    allowed = [e for g in sorted(groups) for e in range(g * G, (g + 1) * G)]
    sub = [keys_row[e] for e in allowed]
    picked = _brute_topk(sub, k)
    return [allowed[i] for i in picked]


@pytest.mark.parametrize("E,k,n_group,topk_group", [(8, 2, 4, 2), (12, 3, 3, 1), (8, 4, 2, 2),
                                                    (16, 4, 8, 3), (6, 2, 6, 4)])
def test_grouped_routing_matches_brute_force(E, k, n_group, topk_group):
    rng = np.random.default_rng(50 + E + k)
    for trial in range(40):
        if trial % 4 == 0:
            logits = (rng.integers(-2, 3, size=(1, E)) / 2.0).astype(F32)   # ties
        else:
            logits = rng.standard_normal((1, E)).astype(F32)
        bias = (rng.standard_normal(E) * 0.1).astype(F32)
        idx, w = orc.route_grouped(logits, bias, k, 2.5, n_group, topk_group)
        keys = orc.selection_keys(orc.sigmoid_scores(logits), bias)[0].tolist()
        assert idx[0].tolist() == _brute_grouped(keys, k, n_group, topk_group)
        assert abs(float(w[0].astype(np.float64).sum()) - 2.5) < 4 * k * 2.4e-7


def test_grouped_routing_degenerate_cases_are_plain_routing():
    rng = np.random.default_rng(77)
    logits = rng.standard_normal((64, 32)).astype(F32)
    bias = (rng.standard_normal(32) * 0.1).astype(F32)
    ref = orc.route(logits, bias, 6, 2.5)
    for n_group, topk_group in [(1, 1), (4, 4), (32, 32)]:
        got = orc.route_grouped(logits, bias, 6, 2.5, n_group, topk_group)
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_grouped_routing_keeps_experts_inside_the_best_groups():
    # group 1 (experts 4..7) has the two best keys; with topk_group = 1 every
    # selected expert must come from it even though expert 0 has a high key
    s = np.array([[0.9, 0.1, 0.1, 0.1, 0.8, 0.85, 0.2, 0.3]], F32)
    logits = np.log(s / (1 - s)).astype(F32)
    idx, w = orc.route_grouped(logits, np.zeros(8, F32), 2, 1.0, 2, 1)
    assert sorted(idx[0].tolist()) == [4, 5]
    idx2, _ = orc.route_grouped(logits, np.zeros(8, F32), 2, 1.0, 2, 2)
    assert idx2[0].tolist() == [0, 5]
