"""The oracle's temperature / top-p sampler pinned to its definition.

Pins, each of which a plausible slip (a dropped temperature, a reversed sort,
an unstable tie order, an off-by-one nucleus, a sample drawn in sorted order
instead of token-id order) fails:
* hand-worked cases (tests/golden/top_p_hand_worked.json);
* with top_p = 1 the inverse CDF over a fine grid of u reproduces the softmax
  of l / T computed by scipy, token by token;
* with top_p < 1 the grid hits exactly the nucleus, each token in proportion
  to its probability renormalised over the nucleus;
* the nucleus is the smallest set of that mass (brute force over every subset
  of tiny rows) and the most probable one of that size;
* the nucleus equals the set kept by transformers' top-p logits warper away
  from its boundary;
* greedy limits: T -> 0 and top_p -> 0 give the argmax, lowest id on ties.
"""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.special

from oracle import sample as osample

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "top_p_hand_worked.json")) as fh:
    GOLDEN = json.load(fh)


def _rows(n, v, sigma, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, v)) * sigma).astype(np.float32)


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=lambda c: c["name"])
def test_hand_worked(case):
    s = osample.sample_top_p(np.array(case["logits"], np.float32), case["T"], case["top_p"], case["u"])
    assert s.token == case["token"], case["why"]
    assert s.nucleus == case["nucleus"], case["why"]


def _grid_counts(logits, T, top_p, n):
    counts = np.zeros(logits.size, np.int64)
    for i in range(n):
        counts[osample.sample_top_p(logits, T, top_p, (i + 0.5) / n).token] += 1
    return counts


@pytest.mark.parametrize("T", [1.0, 0.7, 2.5])
def test_full_vocab_frequencies_are_the_softmax(T):
    l = _rows(1, 24, 1.5, 11)[0]
    n = 20000
    counts = _grid_counts(l, T, 1.0, n)
    p = scipy.special.softmax(l.astype(np.float64) / T)
    # a uniform grid through an inverse CDF lands n * p_t (+- 1) times on token t
    assert np.all(np.abs(counts - n * p) <= 1.0 + 1e-6), np.abs(counts - n * p).max()


def test_nucleus_frequencies_are_renormalised():
    l = _rows(1, 20, 1.0, 12)[0]
    top_p, T, n = 0.6, 0.8, 20000
    counts = _grid_counts(l, T, top_p, n)
    p = scipy.special.softmax(l.astype(np.float64) / T)
    order = np.argsort(-p, kind="stable")
    k = int(np.searchsorted(np.cumsum(p[order]), top_p)) + 1
    nucleus = set(order[:k].tolist())
    assert set(np.flatnonzero(counts).tolist()) == nucleus
    pn = np.where(np.isin(np.arange(l.size), list(nucleus)), p, 0.0)
    pn /= pn.sum()
    assert np.all(np.abs(counts - n * pn) <= 1.0 + 1e-6)


@pytest.mark.parametrize("seed", range(6))
def test_nucleus_is_the_smallest_set_brute_force(seed):
    v = 7
    l = _rows(1, v, 1.2, 100 + seed)[0]
    if seed == 5:
        l[2] = l[4] = l[6]  # ties
    for top_p in (0.05, 0.3, 0.5, 0.77, 0.9, 0.99):
        s = osample.sample_top_p(l, 1.0, top_p, 0.5)
        q = osample.masses(l, 1.0)
        need = s.need
        best = None
        for size in range(1, v + 1):
            reach = [c for c in itertools.combinations(range(v), size) if int(q[list(c)].sum()) >= need]
            if reach:
                best = (size, max(int(q[list(c)].sum()) for c in reach))
                break
        assert (s.nucleus, s.nucleus_mass) == best, (top_p, s, best)


def test_nucleus_matches_transformers_warper():
    torch = pytest.importorskip("torch")
    lp = pytest.importorskip("transformers.generation.logits_process")
    rows = _rows(12, 3000, 2.0, 13)
    checked = 0
    for r, top_p, T in itertools.product(range(rows.shape[0]), (0.5, 0.9), (1.0, 0.6)):
        l = rows[r]
        s = osample.sample_top_p(l, T, top_p, 0.25)
        q = osample.masses(l, T)
        order = np.argsort(-l.astype(np.float64), kind="stable")
        cum = np.cumsum(q[order].astype(np.float64)) / float(s.total_mass)
        k = s.nucleus
        if abs(cum[k - 1] - top_p) < 1e-6 or (k > 1 and abs(cum[k - 2] - top_p) < 1e-6):
            continue  # too close to the boundary for the warper's own rounding
        warp = lp.TopPLogitsWarper(top_p)
        kept = torch.isfinite(warp(None, torch.tensor(l.astype(np.float64) / T)[None]))[0].numpy()
        assert set(np.flatnonzero(kept).tolist()) == set(order[:k].tolist())
        checked += 1
    assert checked >= 20


@pytest.mark.parametrize("seed", range(4))
def test_greedy_limits(seed):
    l = _rows(1, 500, 1.0, 200 + seed)[0]
    if seed == 3:
        l[7] = l[300] = l.max() + 1.0  # tie at the top: lowest id wins
    g = osample.greedy(l)
    assert g == int(np.argmax(l))
    for u in (0.0, 0.5, 0.999):
        assert osample.sample_top_p(l, 0.0, 0.9, u).token == g
        assert osample.sample_top_p(l, -1.0, 0.9, u).token == g
        assert osample.sample_top_p(l, 1.0, 0.0, u).token == g
        cold = osample.sample_top_p(l, 1e-3, 0.95, u).token
        if seed == 3:  # two tokens share the top mass: the draw picks either
            assert cold in (7, 300)
        else:
            assert cold == g


def test_ties_at_the_boundary_enter_by_lower_id():
    """100 tokens of logit 1 scattered among 900 of logit 0; top_p chosen so that
    the nucleus takes the 100 and exactly 50 of the tied ones: the 50 lowest ids."""
    rng = np.random.default_rng(15)
    l = np.zeros(1000, np.float32)
    high = rng.choice(1000, 100, replace=False)
    l[high] = 1.0
    e = float(np.exp(np.float64(1.0)))
    top_p = (100 * e + 49.5) / (100 * e + 900)
    low = np.setdiff1d(np.arange(1000), high)[:50]
    expect = set(high.tolist()) | set(low.tolist())
    n = 40000
    counts = _grid_counts(l, 1.0, top_p, n)
    assert set(np.flatnonzero(counts).tolist()) == expect
    assert osample.sample_top_p(l, 1.0, top_p, 0.5).nucleus == 150


def test_draw_covers_the_nucleus_in_id_order():
    """u = 0 draws the lowest nucleus id, u just below 1 the highest."""
    l = _rows(1, 300, 1.0, 14)[0]
    s0 = osample.sample_top_p(l, 1.0, 0.7, 0.0)
    s1 = osample.sample_top_p(l, 1.0, 0.7, np.nextafter(1.0, 0.0))
    order = np.argsort(-l.astype(np.float64), kind="stable")[:s0.nucleus]
    assert s0.token == int(order.min()) and s1.token == int(order.max())


def test_rejects_bad_inputs():
    l = np.zeros(4, np.float32)
    for bad in (lambda: osample.sample_top_p(l, 1.0, 0.5, 1.0),
                lambda: osample.sample_top_p(l, 1.0, 0.5, -0.1),
                lambda: osample.sample_top_p(np.array([0.0, np.nan], np.float32), 1.0, 0.5, 0.1),
                lambda: osample.sample_top_p(np.zeros(0, np.float32), 1.0, 0.5, 0.1)):
        with pytest.raises(ValueError):
            bad()


def test_margin_ignores_forced_nucleus_boundaries():
    """top_p 0 keeps one token and top_p 1 all of them whatever the masses'
    rounding: only the draw's own boundary bounds the margin there."""
    l = _rows(1, 400, 1.0, 16)[0]
    for top_p in (0.0, 1.0):
        s = osample.sample_top_p(l, 1.0, top_p, 0.37)
        assert s.margin > 0
    s = osample.sample_top_p(l, 1.0, 0.8, 0.37)
    assert 1 < s.need < s.total_mass and s.margin > 0


def test_largest_row_sums_without_overflow():
    """At the largest vocabulary, equal logits give Q = 2^17 * 2^46 = 2^63 exactly:
    the 64-bit sums hold the worst case, and every token is equally likely."""
    l = np.zeros(osample.MAX_VOCAB, np.float32)
    s = osample.sample_top_p(l, 1.0, 1.0, 0.5)
    assert s.total_mass == 1 << 63 and s.nucleus == osample.MAX_VOCAB
    assert s.token == osample.MAX_VOCAB // 2
    s = osample.sample_top_p(l, 1.0, 0.25, 0.5)
    assert s.nucleus == osample.MAX_VOCAB // 4 and s.token == osample.MAX_VOCAB // 8
    with pytest.raises(ValueError):
        osample.sample_top_p(np.zeros(osample.MAX_VOCAB + 1, np.float32), 1.0, 0.5, 0.5)


def test_fixed_point_nucleus_is_the_real_valued_one():
    """The fixed-point decisions (masses rounded to 2^-46, integer sums) give
    the nucleus and the token that exact real arithmetic on the same fp64
    probabilities gives, wherever the real boundary is not within the
    quantisation's reach: each mass moves by at most half a unit, so a sum of
    V masses by at most V/2 units (V * 2^-47 in units of the largest p), and
    the fp64 products top_p * Q and u * S add a relative 2^-53 each."""
    from fractions import Fraction

    rng = np.random.default_rng(2024)
    checked = skipped = 0
    for it in range(120):
        V = int(rng.choice([7, 31, 200, 1000]))
        sigma = float(rng.choice([0.3, 1.0, 3.0]))
        T = float(rng.choice([0.5, 1.0, 2.0]))
        top_p = float(rng.choice([0.1, 0.5, 0.9, 0.99]))
        u = float(rng.random())
        l = (rng.standard_normal(V) * sigma).astype(np.float32)
        got = osample.sample_top_p(l, T, top_p, u)
        # exact rationals of the fp64 probabilities (the largest is exactly 1)
        l64 = l.astype(np.float64)
        p = np.exp((l64 - l64.max()) * (1.0 / float(np.float32(T))))
        F = [Fraction(float(x)) for x in p]
        total = sum(F)
        order = np.argsort(-l64, kind="stable")
        need = Fraction(float(np.float32(top_p))) * total
        cum, k = Fraction(0), None
        cums = []
        for j, t in enumerate(order):
            cum += F[t]
            cums.append(cum)
            if k is None and cum >= need:
                k = j + 1
        eps = Fraction(V, 2 ** 47) + total * Fraction(1, 2 ** 52)
        near = abs(cums[k - 1] - need) <= eps or (k >= 2 and abs(cums[k - 2] - need) <= eps)
        if near:
            skipped += 1
            continue
        assert got.nucleus == k, (it, got.nucleus, k)
        S = cums[k - 1]
        y = Fraction(u) * S
        acc, tok, gap = Fraction(0), None, None
        for t in sorted(int(x) for x in order[:k]):
            lo, acc = acc, acc + F[t]
            if tok is None and acc > y:
                tok, gap = t, min(y - lo, acc - y)
        if gap <= eps + S * Fraction(1, 2 ** 52):
            skipped += 1
            continue
        assert got.token == tok, (it, got.token, tok)
        checked += 1
    assert checked >= 100 and skipped <= 20, (checked, skipped)
