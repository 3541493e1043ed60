"""Pins of the oracle's anchor-adaptive selection (mode "topp_anchor").

"Claude Opus 长上下文 KV Cache 稀疏注意力", §多上下文场景下的跨文档注意力恢复: the sink
and local blocks are anchors; the scores' bounds (max, min) set the Top-P
ratio, higher when the maximum stands well above the anchors.  Reading taken
(no formula on the page): a = the anchors' best score, hi / lo = the middle
blocks' best / worst, r = clamp((hi - a) / (hi - lo), 0, 1), ratio =
min_ratio + r (max_ratio - min_ratio), k_max = floor(ratio n_mid), then
top-p with that cap.  The pins: the anchors' scores by the linearity identity,
the cap against the formula written out here and the kept set against
brute-force enumeration, the two clamped ends, the degenerate ratio range
(= plain top-p) and monotonicity in the anchor score.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_kv_spattn_b200.workloads import make_inputs
from cases import SMALL_ANCHOR
from oracle.marshal import dequant, run_oracle
from test_oracle_pins import _brute_topp, _select_rows

pytestmark = pytest.mark.filterwarnings("ignore")


def test_anchor_mode_scores_the_anchor_blocks():
    """Sink and local blocks get q_bar . K_bar / sqrt(d) = the mean token logit
    too; columns past the sequence stay -inf."""
    w = SMALL_ANCHOR
    inp = make_inputs(w)
    res = run_oracle(inp)
    K = dequant(inp, "k")
    q = inp["q"].to(torch.float64)
    P, H, G = w.block_size, w.num_kv_heads, w.num_q_heads // w.num_kv_heads
    scale = 1.0 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        nb = (L + P - 1) // P
        for h in range(H):
            s = res["scores"][b, 0, h]
            for j in list(range(w.sink_blocks)) + list(range(nb - w.local_blocks, nb)):
                page = int(inp["block_table"][b, j])
                n = min(P, L - j * P)
                logits = q[b, 0, h * G:(h + 1) * G] @ K[page, h, :n].T * scale
                assert s[j] == pytest.approx(float(logits.mean()), rel=1e-12, abs=1e-12)
            assert np.all(s[nb:] == -np.inf)


def _cap(a, hi, lo, n, mn, mx):
    r = (hi - a) / (hi - lo) if hi > lo else 0.0
    r = min(max(r, 0.0), 1.0)
    return min(n, math.floor((mn + r * (mx - mn)) * n))


def _anchor_row(S, anchors_sink, mid, anchors_local):
    return list(anchors_sink) + list(mid) + list(anchors_local)


@pytest.mark.parametrize("seed", range(40))
def test_anchor_cap_matches_formula_and_brute_force(seed):
    rng = np.random.default_rng(500 + seed)
    S, W = 1, 2
    n_mid = int(rng.integers(2, 11))
    mid = rng.normal(scale=2.0, size=n_mid)
    anchors = rng.normal(scale=2.0, size=S + W) + float(rng.choice([-3.0, 0.0, 3.0]))
    p = float(rng.choice([0.5, 0.8, 0.9, 1.0]))
    mn, mx = sorted(float(x) for x in rng.choice([0.1, 0.2, 0.3, 0.5, 0.7], size=2, replace=False))
    k_max = _cap(float(anchors.max()), float(mid.max()), float(mid.min()), n_mid, mn, mx)
    x = (mn + min(max((mid.max() - anchors.max()) / (mid.max() - mid.min()), 0.0), 1.0) * (mx - mn)) * n_mid
    if abs(x - round(x)) < 1e-9:
        pytest.skip("cap lands on an integer within rounding")
    e = np.exp(mid - mid.max())
    prob = np.sort(e / e.sum())[::-1]
    if np.min(np.abs(np.cumsum(prob) - p)) < 1e-9 and p < 1.0:
        pytest.skip("mass lands on p within rounding")
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp_anchor", top_p=p, max_ratio=mx,
                        min_ratio=mn)
    got, _ = _select_rows([_anchor_row(S, anchors[:S], mid, anchors[S:])], S + n_mid + W, prm)
    kept_mid, m_star = _brute_topp(list(mid), p, k_max)
    want = sorted({0} | {S + j for j in kept_mid} | {S + n_mid, S + n_mid + 1})
    assert got == want
    assert len(kept_mid) == min(m_star, k_max)


def test_anchor_clamped_ends():
    """Anchors above the middle's best: min_ratio decides; below its worst:
    max_ratio decides (p = 1 so the cap always binds)."""
    S, W, n = 1, 2, 20
    mid = np.linspace(-1.0, 1.0, n)
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp_anchor", top_p=1.0, max_ratio=0.5,
                        min_ratio=0.1)
    high = _anchor_row(S, [5.0], mid, [0.0, 0.0])
    low = _anchor_row(S, [-5.0], mid, [-6.0, -7.0])
    got_hi, mg_hi = _select_rows([high], S + n + W, prm)
    got_lo, mg_lo = _select_rows([low], S + n + W, prm)
    assert len(got_hi) == S + W + math.floor(0.1 * n)
    assert len(got_lo) == S + W + math.floor(0.5 * n)
    # the kept middle blocks are the best ones
    assert got_hi[S:-W] == list(range(S + n - 2, S + n))
    assert mg_hi > 0 and mg_lo > 0


def test_anchor_equal_ratios_is_plain_topp():
    rng = np.random.default_rng(7)
    S, W, n = 1, 2, 30
    mid = rng.normal(size=n)
    row = _anchor_row(S, [rng.normal()], mid, rng.normal(size=W))
    a = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp_anchor", top_p=0.9, max_ratio=0.3,
                      min_ratio=0.3)
    b = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp", top_p=0.9, max_ratio=0.3)
    plain = [-np.inf] * S + list(mid) + [-np.inf] * W
    assert _select_rows([row], S + n + W, a)[0] == _select_rows([plain], S + n + W, b)[0]


def test_anchor_count_falls_as_the_anchor_rises():
    S, W, n = 1, 2, 40
    mid = np.random.default_rng(3).normal(size=n)
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp_anchor", top_p=1.0, max_ratio=0.6,
                        min_ratio=0.05)
    counts = []
    for a in np.linspace(mid.min() - 1, mid.max() + 1, 25):
        got, _ = _select_rows([_anchor_row(S, [a], mid, [a - 10, a - 10])], S + n + W, prm)
        counts.append(len(got))
    assert all(x >= y for x, y in zip(counts, counts[1:]))
    assert counts[0] == S + W + math.floor(0.6 * n) and counts[-1] == S + W + math.floor(0.05 * n)


def test_anchor_margin_small_when_the_cap_sits_on_an_integer():
    """A cap ratio * n_mid that is an integer is a decision boundary: the
    reported margin is ~0, so parity replays instead of comparing exactly."""
    S, W, n = 1, 2, 10
    mid = np.linspace(0.0, 1.0, n)                 # hi = 1, lo = 0
    # a = 0.5 -> r = 0.5 -> ratio = 0.1 + 0.5 * 0.4 = 0.3 -> 3.0 exactly
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp_anchor", top_p=1.0, max_ratio=0.5,
                        min_ratio=0.1)
    got, mg = _select_rows([_anchor_row(S, [0.5], mid, [0.0, 0.0])], S + n + W, prm)
    assert len(got) == S + W + 3
    assert mg < 1e-9
