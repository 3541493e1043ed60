"""Pins of the oracle's decision margin (CPU only).

The margin decides, row by row, whether the GPU's selection must equal the
oracle's bit for bit (margin > 1e-4) or is checked by replay on the GPU's own
scores.  It is the distance from the inputs to the nearest point where the
kept set changes, on each quantity the selection decides on:

* the score gap across the cut: the worst kept middle block against the best
  dropped one (score units);
* for top-p, the distance of the threshold p to the nearest value p' at which
  the kept set differs (probability units).

Here both are found by enumeration on rows of at most 10 middle blocks, with
no sorting and no prefix sums: the kept set comes from a brute-force search
over all subsets, the cut gap from all (kept, dropped) pairs, and the
breakpoints in p from the largest mass of any i blocks, where the brute-force
selection is re-run at every candidate p'.  The oracle's margin must equal
that value.  A margin that is always 0, or that drops any of the terms, fails
here; so does a margin that is larger than the true distance, which would let
a near-tie through as "exact".  A second test checks the property the
parity tests rely on: perturbing every score by less than a third of the
margin never changes the oracle's selection.

Source of the rules: "Claude Opus 长上下文 KV Cache 稀疏注意力" §稀疏注意力与 KV Cache
压缩的工程实现 (Top-P block selection), "CSA + HCA 混合注意力机制" §4.2 (top-k over
scored entries); ties rank the lower block index first.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import pytest

import oracle

INF = math.inf


def _probs(s):
    e = np.exp(np.asarray(s, dtype=np.float64) - max(s))
    return e / e.sum()


def _lex_best(subsets, key):
    best = max(key(T) for T in subsets)
    return frozenset(min(sorted(T) for T in subsets if key(T) == best))


def _bf_topk(s, k):
    """The k-subset with the largest score sum, lexicographically first."""
    n = len(s)
    if k <= 0:
        return frozenset()
    return _lex_best(list(itertools.combinations(range(n), min(k, n))), lambda T: math.fsum(s[j] for j in T))


def _bf_topp(s, p, k_max):
    """Smallest cardinality m with a subset of mass >= p, then the best such
    subset; above k_max the k_max blocks of largest score instead."""
    prob = _probs(s)
    n = len(s)
    for m in range(1, n + 1):
        subs = [T for T in itertools.combinations(range(n), m)
                if m == n or math.fsum(prob[j] for j in T) >= p]
        if subs:
            break
    if m > k_max:
        return _bf_topk(s, k_max)
    return _lex_best(subs, lambda T: math.fsum(prob[j] for j in T))


def _bf_keep(s, mode, p, k, k_max):
    if mode == "topk":
        return _bf_topk(s, min(k if k > 0 else k_max, k_max))
    return _bf_topp(s, p, k_max)


def _bf_margin(s, mode, p, k, k_max):
    n = len(s)
    M = _bf_keep(s, mode, p, k, k_max)
    dropped = set(range(n)) - M
    gap = min((s[i] - s[j] for i in M for j in dropped), default=INF)
    if mode == "topk":
        return gap
    prob = _probs(s)
    # the kept set can only change where p' equals the largest mass of some
    # number of blocks (or just above it)
    C = [max(math.fsum(prob[j] for j in T) for T in itertools.combinations(range(n), i))
         for i in range(1, n)]
    down = [p - c for c in C if 0.0 < c < p and _bf_topp(s, c, k_max) != M]
    up = [c - p for c in C if p <= c and c + 1e-12 <= 1.0 and _bf_topp(s, c + 1e-12, k_max) != M]
    return min([gap] + down + up)


def _oracle_row(s, mode, p, k, ratio):
    S, W = 1, 2
    n = len(s)
    nb = S + n + W
    dims = oracle.Dims(batch=1, q_tokens=1, num_q_heads=1, num_kv_heads=1, head_dim=128,
                       block_size=64, num_pages=nb, max_blocks=nb, max_sel=nb)
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode=mode, top_k=k, top_p=p, max_ratio=ratio)
    row = np.full((1, 1, 1, nb), -np.inf)
    row[0, 0, 0, S:S + n] = s
    sel, cnt, mg = oracle.select(dims, prm, row, np.array([nb * 64], np.int32))
    kept = frozenset(int(j) - S for j in sel[0, 0, :cnt[0, 0]] if S <= j < S + n)
    return kept, float(mg[0, 0])


def _case(seed):
    """A small row: random or integer scores, top-k or top-p, capped or not."""
    rng = np.random.default_rng(7000 + seed)
    n = int(rng.integers(1, 11))
    if seed % 4 == 0:
        s = rng.integers(-2, 3, size=n).astype(float)            # many exact ties
    else:
        s = rng.normal(scale=float(rng.choice([0.5, 1.0, 2.0])), size=n)
    mode = "topk" if seed % 2 == 0 else "topp"
    ratio = float(rng.choice([0.0, 0.3, 0.5, 0.8]))
    k_max = min(n, int(math.floor(ratio * n))) if ratio > 0 else n
    k = int(rng.integers(0, n + 1)) if mode == "topk" else 0
    if mode == "topk" and k == 0 and ratio == 0.0:
        ratio, k_max = 1.0, n
    p = float(rng.choice([0.3, 0.5, 0.7, 0.9, 0.95, 1.0]))
    return [float(x) for x in s], mode, p, k, ratio, k_max


@pytest.mark.parametrize("seed", range(120))
def test_margin_equals_enumerated_distance(seed):
    s, mode, p, k, ratio, k_max = _case(seed)
    kept, mg = _oracle_row(s, mode, p, k, ratio)
    assert kept == _bf_keep(s, mode, p, k, k_max)
    want = _bf_margin(s, mode, p, k, k_max)
    if want == INF:
        assert mg == INF
    else:
        assert mg == pytest.approx(want, rel=1e-9, abs=1e-12), (s, mode, p, k, ratio)


def test_margin_terms_each_bind():
    """Hand rows where each term of the margin is the smallest: the score gap
    at the cut, p above the previous prefix mass, the next prefix mass above
    p, and (capped) p above the mass of k_max - 1 blocks."""
    # probabilities 0.5, 0.25, 0.125, 0.0625, ... (scores log 2^-i)
    s = [math.log(2.0 ** -i) for i in range(6)]
    prob = _probs(s)
    C = np.cumsum(prob)
    # uncapped, p just above C_2: m* = 3; p - C_2 is the smallest term
    p = float(C[1] + 1e-3)
    kept, mg = _oracle_row(s, "topp", p, 0, 0.0)
    assert kept == {0, 1, 2} and mg == pytest.approx(1e-3, rel=1e-9)
    # uncapped, p just below C_3: C_3 - p is the smallest term
    p = float(C[2] - 2e-3)
    kept, mg = _oracle_row(s, "topp", p, 0, 0.0)
    assert kept == {0, 1, 2} and mg == pytest.approx(2e-3, rel=1e-9)
    # the same row with its cut inside a near tie: the score gap binds
    s2 = list(s)
    s2[3] = s2[2] - 1e-6
    kept, mg = _oracle_row(s2, "topp", 0.8, 0, 0.0)
    assert kept == {0, 1, 2} and mg == pytest.approx(1e-6, rel=1e-6)
    # capped at k_max = 2 (ratio 0.4 of 6 blocks), p = 0.8 > C_2 = 0.75...: a
    # p down at C_1 = 0.507... would keep one block
    kept, mg = _oracle_row(s, "topp", 0.8, 0, 0.4)
    assert kept == {0, 1}
    assert mg == pytest.approx(min(0.8 - C[0], s[1] - s[2]), rel=1e-9)
    # m* = 1: no lower p changes the set; m* = n: no gap and no higher p
    kept, mg = _oracle_row([3.0, 0.0, -1.0], "topp", 0.5, 0, 0.0)
    assert kept == {0} and mg == pytest.approx(min(3.0 - 0.0, float(_probs([3.0, 0.0, -1.0])[0]) - 0.5))
    kept, mg = _oracle_row([0.0, 0.0], "topp", 1.0, 0, 0.0)
    assert kept == {0, 1} and mg == pytest.approx(1.0 - 0.5)


@pytest.mark.parametrize("seed", range(60))
def test_perturbations_inside_the_margin_keep_the_set(seed):
    """Moving every score by less than a third of the margin (and p by less
    than the margin) leaves the oracle's kept set as it was: the property
    that makes a margin above the GPU's score error a guarantee of identical
    indices."""
    s, mode, p, k, ratio, k_max = _case(seed)
    kept, mg = _oracle_row(s, mode, p, k, ratio)
    if not (mg > 1e-9) or mg == INF:
        mg = 1.0 if mg == INF else mg
        if mg <= 1e-9:
            pytest.skip("the cut sits on a tie: no perturbation is safe")
    rng = np.random.default_rng(9000 + seed)
    for _ in range(20):
        d = rng.uniform(-1.0, 1.0, size=len(s)) * min(mg, 1.0) / 3.0
        moved = [x + y for x, y in zip(s, d)]
        assert _oracle_row(moved, mode, p, k, ratio)[0] == kept
        if mode == "topp":
            e = float(rng.uniform(-1.0, 1.0)) * min(mg, 1.0) * 0.99
            p2 = min(1.0, max(1e-6, p + e))
            assert _oracle_row(s, mode, p2, k, ratio)[0] == kept
