"""Pins of the float64 oracle against things other than itself.

Each test pins one step of the oracle to an independent fact: a library
routine (torch dtype conversions, torch/numpy reductions, torch SDPA), a
closed form, an identity that holds by linearity, or brute-force enumeration
over every subset on tiny inputs.  They run on the CPU only.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_kv_spattn_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle.marshal import bits16, dequant, dims_of, host_arrays, params_of, run_oracle

from tests.cases import SMALL_FP8_CHUNK, SMALL_RAGGED, SMALL_TOPP


@pytest.fixture(scope="module")
def tiny():
    return make_inputs(WORKLOADS["tiny_4k_gqa4"])


# --------------------------------------------------------------- decoding

def test_bf16_decoding_matches_torch_for_every_code():
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decoding_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert nan.sum() == 2                      # S.1111.111 only: no infinities
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------ compression

@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED], ids=lambda w: w.name)
def test_compress_is_mean_of_filled_tokens(w):
    inp = make_inputs(w)
    a = host_arrays(inp)
    kbar = oracle.compress_keys(dims_of(inp), a["k_cache"], a["k_scale"], a["block_table"],
                                a["seq_lens"])
    K = dequant(inp, "k")
    P = w.block_size
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        for j in range((L + P - 1) // P):
            page = int(inp["block_table"][b, j])
            n = min(P, L - j * P)
            ref = K[page, :, :n, :].mean(dim=1).numpy()      # torch reduction, float64
            np.testing.assert_allclose(kbar[page], ref, rtol=1e-13, atol=1e-13)


def test_compress_constant_block_closed_form():
    inp = make_inputs(SMALL_RAGGED)
    k = inp["k_cache"]
    P = SMALL_RAGGED.block_size
    b, j = 1, 0
    L = int(inp["seq_lens"][b])
    page = int(inp["block_table"][b, j])
    row = torch.linspace(-3, 3, SMALL_RAGGED.head_dim).to(torch.bfloat16)
    k[page, 0, :min(P, L)] = row
    a = host_arrays(inp)
    kbar = oracle.compress_keys(dims_of(inp), a["k_cache"], None, a["block_table"], a["seq_lens"])
    assert np.array_equal(kbar[page, 0], row.to(torch.float64).numpy())


# ----------------------------------------------------------------- scores

@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK], ids=lambda w: w.name)
def test_scores_equal_group_mean_of_token_logits(w):
    """By linearity, q_bar . K_bar / sqrt(d) is the mean over the group's heads
    and the block's tokens of the per-token logits q_i . k / sqrt(d)."""
    inp = make_inputs(w)
    res = run_oracle(inp)
    K = dequant(inp, "k")
    q = inp["q"].to(torch.float64)
    P, H, G = w.block_size, w.num_kv_heads, w.num_q_heads // w.num_kv_heads
    scale = 1.0 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        nb = (L + P - 1) // P
        for t in range(w.q_tokens):
            for h in range(H):
                s = res["scores"][b, t, h]
                for j in range(nb):
                    if j < w.sink_blocks or j >= nb - w.local_blocks:
                        assert s[j] == -np.inf
                        continue
                    page = int(inp["block_table"][b, j])
                    n = min(P, L - j * P)
                    logits = q[b, t, h * G:(h + 1) * G] @ K[page, h, :n].T * scale   # [G, n]
                    assert s[j] == pytest.approx(float(logits.mean()), rel=1e-12, abs=1e-12)
                assert np.all(s[nb:] == -np.inf)


# -------------------------------------------------------------- selection

def _select_rows(scores_rows, n_blocks, params, max_sel=None):
    """Run the oracle's selection on hand-made score rows (one request, one
    KV head, Tq = len(scores_rows))."""
    Tq = len(scores_rows)
    dims = oracle.Dims(batch=1, q_tokens=Tq, num_q_heads=1, num_kv_heads=1, head_dim=128,
                       block_size=64, num_pages=n_blocks, max_blocks=n_blocks,
                       max_sel=max_sel or n_blocks)
    s = np.full((1, Tq, 1, n_blocks), -np.inf)
    for t, row in enumerate(scores_rows):
        s[0, t, 0, :] = row
    sel, cnt, margin = oracle.select(dims, params, s, np.array([n_blocks * 64], np.int32))
    return [int(x) for x in sel[0, 0, :cnt[0, 0]]], float(margin[0, 0])


def _lex_best(subsets, key):
    best = max(key(T) for T in subsets)
    return min(sorted(T) for T in subsets if key(T) == best)


def _brute_topk(s, k):
    mid = range(len(s))
    subs = list(itertools.combinations(mid, k))
    return _lex_best(subs, lambda T: math.fsum(s[j] for j in T))


def _brute_topp(s, p, k_max):
    e = np.exp(np.asarray(s) - max(s))
    prob = e / e.sum()
    n = len(s)
    for m in range(1, n + 1):
        # the whole middle set has mass 1 exactly, whatever the rounding
        subs = [T for T in itertools.combinations(range(n), m)
                if m == n or math.fsum(prob[j] for j in T) >= p]
        if subs:
            break
    if m > k_max:
        return _brute_topk(list(s), k_max), m
    return _lex_best(subs, lambda T: math.fsum(prob[j] for j in T)), m


def _row(S, mid_scores, W):
    return [-np.inf] * S + list(mid_scores) + [-np.inf] * W


@pytest.mark.parametrize("seed", range(40))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    S, W = int(rng.integers(0, 3)), int(rng.integers(0, 3))
    n_mid = int(rng.integers(1, 11))
    s = rng.normal(size=n_mid)
    if seed % 3 == 0:                           # integer scores: many exact ties
        s = rng.integers(-2, 3, size=n_mid).astype(float)
    k = int(rng.integers(0, n_mid + 1))
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topk", top_k=k, max_ratio=0.0)
    if k == 0:
        prm.max_ratio = 1.0                    # k from the ratio: all middle blocks
        k = n_mid
    got, _ = _select_rows([_row(S, s, W)], S + n_mid + W, prm)
    want = sorted(set(range(S)) | {S + j for j in _brute_topk(list(s), k)}
                  | set(range(S + n_mid, S + n_mid + W)))
    assert got == want


@pytest.mark.parametrize("seed", range(40))
def test_topp_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    S, W = 1, 2
    n_mid = int(rng.integers(1, 11))
    s = rng.normal(scale=2.0, size=n_mid)
    p = float(rng.choice([0.3, 0.5, 0.7, 0.9, 0.95, 1.0]))
    ratio = float(rng.choice([0.0, 0.3, 0.5]))
    k_max = int(math.floor(ratio * n_mid)) if ratio > 0 else n_mid
    e = np.exp(s - s.max())
    prob = np.sort(e / e.sum())[::-1]
    if np.min(np.abs(np.cumsum(prob) - p)) < 1e-9 and p < 1.0:
        pytest.skip("mass lands on p within rounding")
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topp", top_p=p, max_ratio=ratio)
    got, _ = _select_rows([_row(S, s, W)], S + n_mid + W, prm)
    mid, m_star = _brute_topp(list(s), p, k_max)
    want = sorted({0} | {S + j for j in mid} | {S + n_mid, S + n_mid + 1})
    assert got == want
    assert len(mid) == min(m_star, k_max)


def test_topp_minimal_prefix_and_cap():
    # probabilities 0.5, 0.25, 0.125, ...: with p = 0.8 the minimal prefix is 3
    s = [math.log(2.0 ** -i) for i in range(8)]
    prm = oracle.Params(sink_blocks=1, local_blocks=2, mode="topp", top_p=0.8, max_ratio=0.0)
    got, _ = _select_rows([_row(1, s, 2)], 11, prm)
    assert got == [0, 1, 2, 3, 9, 10]
    prm.max_ratio = 0.25                        # k_max = floor(0.25 * 8) = 2 < 3
    got, _ = _select_rows([_row(1, s, 2)], 11, prm)
    assert got == [0, 1, 2, 9, 10]


def test_tie_break_prefers_lower_index():
    s = [1.0, 3.0, 2.0, 3.0, 3.0, 0.0]
    prm = oracle.Params(sink_blocks=1, local_blocks=1, mode="topk", top_k=2)
    got, margin = _select_rows([_row(1, s, 1)], 8, prm)
    assert got == [0, 2, 4, 7]                 # middle j = 1 and 3 (scores 3, 3; 4 loses)
    assert margin == 0.0                        # the cut falls inside a tie


def test_chunk_union_over_tokens():
    s0 = [5.0, 4.0, 0.0, 0.0, 0.0, 0.0]
    s1 = [0.0, 0.0, 0.0, 0.0, 4.0, 5.0]
    prm = oracle.Params(sink_blocks=1, local_blocks=2, mode="topk", top_k=2)
    got, _ = _select_rows([_row(1, s0, 2), _row(1, s1, 2)], 9, prm)
    assert got == [0, 1, 2, 5, 6, 7, 8]


@pytest.mark.parametrize("nb", [1, 2, 3])
def test_short_context_keeps_every_block(nb):
    prm = oracle.Params(sink_blocks=1, local_blocks=2, mode="topk", top_k=4)
    got, _ = _select_rows([[-np.inf] * nb], nb, prm)
    assert got == list(range(nb))


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED,
                               WORKLOADS["tiny_4k_gqa4"]], ids=lambda w: w.name)
def test_selection_invariants(w):
    inp = make_inputs(w)
    res = run_oracle(inp)
    P, S, W = w.block_size, w.sink_blocks, w.local_blocks
    for b in range(w.batch):
        nb = (int(inp["seq_lens"][b]) + P - 1) // P
        n_mid = max(0, nb - S - W)
        k_max = math.floor(w.max_ratio * n_mid) if w.max_ratio > 0 else n_mid
        k = min(w.top_k if (w.mode == "topk" and w.top_k > 0) else k_max, k_max)
        for h in range(w.num_kv_heads):
            sel = list(res["sel_idx"][b, h, :res["sel_count"][b, h]])
            assert sel == sorted(set(sel))
            assert set(range(min(S, nb))) | set(range(max(0, nb - W), nb)) <= set(sel)
            mid = [j for j in sel if S <= j < nb - W]
            if w.mode == "topk":
                per_token = len(mid) if w.q_tokens == 1 else None
                if per_token is not None:
                    assert per_token == k
                assert k <= len(mid) <= min(n_mid, w.q_tokens * k)
            else:
                assert len(mid) <= k_max


def test_kept_fraction_is_the_ratio_when_the_cap_binds():
    inp = make_inputs(SMALL_TOPP)
    res = run_oracle(inp)
    nb = (SMALL_TOPP.seq_len + 63) // 64
    n_mid = nb - 3
    for b in range(SMALL_TOPP.batch):
        for h in range(SMALL_TOPP.num_kv_heads):
            assert res["sel_count"][b, h] == 3 + math.floor(0.15 * n_mid)


def test_planted_blocks_are_recalled(tiny):
    res = run_oracle(tiny)
    for h in range(2):
        sel = set(res["sel_idx"][0, h, :res["sel_count"][0, h]].tolist())
        assert set(tiny["boosted"][0][h].tolist()) <= sel
        assert res["sel_count"][0, h] == 1 + 2 + 8


# -------------------------------------------------------------- attention

def _sdpa_reference(inp, keep_mask_fn=None):
    """torch SDPA in float64 over every stored token, with a boolean mask of
    visible tokens: position < L, position <= the query's position, and (if
    given) the token's block kept for the (b, h) unit."""
    w = inp["workload"]
    K, V = dequant(inp, "k"), dequant(inp, "v")
    q = inp["q"].to(torch.float64)
    P, H, G, Tq = w.block_size, w.num_kv_heads, w.num_q_heads // w.num_kv_heads, w.q_tokens
    out = torch.zeros_like(q)
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        nb = (L + P - 1) // P
        pages = inp["block_table"][b, :nb].long()
        kb = K[pages].permute(1, 0, 2, 3).reshape(H, nb * P, -1)     # [H, nb*P, d]
        vb = V[pages].permute(1, 0, 2, 3).reshape(H, nb * P, -1)
        kb = torch.nan_to_num(kb)                                     # tail slots are masked
        vb = torch.nan_to_num(vb)
        pos = torch.arange(nb * P)
        qpos = L - Tq + torch.arange(Tq)
        vis = (pos[None, :] < L) & (pos[None, :] <= qpos[:, None])    # [Tq, nb*P]
        for h in range(H):
            m = vis.clone()
            if keep_mask_fn is not None:
                m &= keep_mask_fn(b, h)[pos // P][None, :]
            qq = q[b, :, h * G:(h + 1) * G].permute(1, 0, 2)           # [G, Tq, d]
            o = torch.nn.functional.scaled_dot_product_attention(
                qq, kb[h].expand(G, -1, -1), vb[h].expand(G, -1, -1),
                attn_mask=m.expand(G, -1, -1))
            out[b, :, h * G:(h + 1) * G] = o.permute(1, 0, 2)
    return out.numpy()


SELECT_ALL = dict(mode="topk", top_k=0, max_ratio=1.0)


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED], ids=lambda w: w.name)
def test_select_all_equals_dense_attention(w):
    inp = make_inputs(w)
    res = run_oracle(inp, params=params_of(w, **SELECT_ALL))
    ref = _sdpa_reference(inp)
    assert np.all(np.isfinite(res["out"]))     # NaN tail slots were never read
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, WORKLOADS["tiny_4k_gqa4"]],
                         ids=lambda w: w.name)
def test_sparse_attention_equals_masked_sdpa(w):
    inp = make_inputs(w)
    res = run_oracle(inp)
    nbmax = inp["max_blocks"]

    def keep(b, h):
        m = torch.zeros(nbmax, dtype=torch.bool)
        m[torch.from_numpy(res["sel_idx"][b, h, :res["sel_count"][b, h]]).long()] = True
        return m

    ref = _sdpa_reference(inp, keep)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


LONG_CHUNK = Workload("long_chunk", batch=1, q_tokens=200, num_q_heads=8, num_kv_heads=2,
                      seq_len=64 * 20 + 9, structure="zipf", mode="topk", max_ratio=0.3, seed=31)


def test_long_chunk_is_causal_everywhere():
    """A chunk longer than the local window (200 tokens against 2 x 64): its
    early tokens must not see the later tokens of middle blocks either, so the
    causal mask applies to every kept block, selected or all."""
    inp = make_inputs(LONG_CHUNK)
    res = run_oracle(inp, params=params_of(LONG_CHUNK, **SELECT_ALL))
    np.testing.assert_allclose(res["out"], _sdpa_reference(inp), rtol=1e-10, atol=1e-12)
    res = run_oracle(inp)
    nbmax = inp["max_blocks"]

    def keep(b, h):
        m = torch.zeros(nbmax, dtype=torch.bool)
        m[torch.from_numpy(res["sel_idx"][b, h, :res["sel_count"][b, h]]).long()] = True
        return m

    np.testing.assert_allclose(res["out"], _sdpa_reference(inp, keep), rtol=1e-10, atol=1e-12)


def test_two_token_closed_form():
    """One request of 2 tokens, one head: out = (e^a v1 + e^b v2) / (e^a + e^b)."""
    w = Workload("two", batch=1, q_tokens=1, num_q_heads=1, num_kv_heads=1, seq_len=2,
                 structure="none", mode="topk", top_k=1, contiguous=True, seed=3)
    inp = make_inputs(w)
    q = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16)
    q[..., 0] = 2.0
    inp["q"] = q
    k = inp["k_cache"]
    k[0, 0, 0] = 0.0
    k[0, 0, 1] = 0.0
    k[0, 0, 0, 0] = 1.0
    k[0, 0, 1, 0] = -1.0
    a, bb = 2.0 / math.sqrt(128), -2.0 / math.sqrt(128)
    v1 = inp["v_cache"][0, 0, 0].to(torch.float64).numpy()
    v2 = inp["v_cache"][0, 0, 1].to(torch.float64).numpy()
    want = (math.exp(a) * v1 + math.exp(bb) * v2) / (math.exp(a) + math.exp(bb))
    res = run_oracle(inp)
    np.testing.assert_allclose(res["out"][0, 0, 0], want, rtol=1e-14, atol=1e-14)


def test_empty_request_gives_zero_output():
    w = SMALL_RAGGED
    inp = make_inputs(w)
    inp["seq_lens"] = inp["seq_lens"].clone()
    inp["seq_lens"][1] = 0
    res = run_oracle(inp)
    assert res["sel_count"][1, 0] == 0
    assert np.all(res["out"][1] == 0.0)


def test_units_subset_matches_full():
    inp = make_inputs(SMALL_TOPP)
    full = run_oracle(inp)
    part = run_oracle(inp, units=[(1, 0)])
    G = SMALL_TOPP.num_q_heads // SMALL_TOPP.num_kv_heads
    np.testing.assert_array_equal(part["out"][1, :, :G], full["out"][1, :, :G])
    assert np.all(part["out"][0] == 0.0)


def test_topp_threshold_is_inclusive():
    """Four equal middle scores give probabilities of exactly 1/4 each; with
    p = 0.5 the minimal prefix reaching p has 2 blocks (mass == p counts), and
    the tie goes to the lower indices."""
    prm = oracle.Params(sink_blocks=1, local_blocks=2, mode="topp", top_p=0.5, max_ratio=0.0)
    got, margin = _select_rows([_row(1, [0.0] * 4, 2)], 7, prm)
    assert got == [0, 1, 2, 5, 6]
    assert margin == 0.0
