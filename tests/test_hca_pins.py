"""Pins of the oracle's weight-free HCA branch.

"CSA + HCA 混合注意力机制" §5.1-5.2: every 128 consecutive tokens are pooled into
one entry and each query attends densely over all entries.  Readings: mean
pooling (the page's pooling is learned), an entry is visible to a query when
all its tokens are at or before the query's position, no position tag and no
sink logit; the branch's output joins the sparse branch's by their
log-sum-exp, which is softmax attention over the union of both key sets.
Pins: the pooled entries against torch means, the dense attention and its
ln-sum-exp against torch's scaled_dot_product_attention and logsumexp, and
the merge of a select-all sparse branch with the HCA branch against one
softmax over the concatenated keys and values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_kv_spattn_b200.workloads import make_inputs
from cases import SMALL_FP8_CHUNK, SMALL_TOPP
from oracle.marshal import dequant, dims_of, host_arrays, params_of

GROUP = 2   # blocks per pooled entry (128 tokens)


def _pool(inp):
    a = host_arrays(inp)
    return oracle.hca_pool(dims_of(inp), a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                           a["block_table"], a["seq_lens"], GROUP)


def _tokens(inp, b, which):
    """float64 [Hkv][L][d]: request b's keys or values in logical order."""
    w = inp["workload"]
    P = w.block_size
    L = int(inp["seq_lens"][b])
    nb = (L + P - 1) // P
    X = dequant(inp, which)
    pages = inp["block_table"][b, :nb].long().cpu()
    return X[pages].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb * P, w.head_dim)[:, :L]


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK], ids=lambda w: w.name)
def test_hca_pool_is_the_group_mean(w):
    inp = make_inputs(w)
    khat, vhat = _pool(inp)
    T = GROUP * w.block_size
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        K, V = _tokens(inp, b, "k"), _tokens(inp, b, "v")
        for g in range(khat.shape[1]):
            if g * T >= L:
                assert not khat[b, g].any() and not vhat[b, g].any()
                continue
            np.testing.assert_allclose(khat[b, g], K[:, g * T:(g + 1) * T].mean(dim=1).numpy(), rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(vhat[b, g], V[:, g * T:(g + 1) * T].mean(dim=1).numpy(), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK], ids=lambda w: w.name)
def test_hca_attend_is_masked_sdpa(w):
    inp = make_inputs(w)
    khat, vhat = _pool(inp)
    a = host_arrays(inp)
    out, lse = oracle.hca_attend(dims_of(inp), params_of(w), a["q"], khat, vhat, a["seq_lens"], GROUP)
    P, G, T = w.block_size, w.num_q_heads // w.num_kv_heads, GROUP * w.block_size
    q = inp["q"].cpu().to(torch.float64)
    scale = 1.0 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        ng = (L + T - 1) // T
        last = torch.tensor([min(L, (g + 1) * T) - 1 for g in range(ng)])
        for t in range(w.q_tokens):
            vis = last <= L - w.q_tokens + t
            for i in range(w.num_q_heads):
                h = i // G
                kk = torch.from_numpy(khat[b, :ng, h])
                vv = torch.from_numpy(vhat[b, :ng, h])
                if not vis.any():
                    assert lse[b, t, i] == -np.inf and not out[b, t, i].any()
                    continue
                ref = torch.nn.functional.scaled_dot_product_attention(
                    q[b, t, i][None, None, None], kk[None, None], vv[None, None],
                    attn_mask=vis[None, None, None], scale=scale)[0, 0, 0]
                np.testing.assert_allclose(out[b, t, i], ref.numpy(), rtol=1e-12, atol=1e-12)
                logits = (kk[vis] @ q[b, t, i]) * scale
                assert lse[b, t, i] == pytest.approx(float(torch.logsumexp(logits, 0)), rel=1e-12, abs=1e-12)


def test_merge_of_branches_is_one_softmax_over_both_key_sets():
    """Sparse branch keeping every block, merged with the HCA branch by
    log-sum-exp, equals SDPA over [all tokens ; pooled entries]."""
    w = SMALL_TOPP.replace(mode="topk", top_k=0, max_ratio=1.0)   # k = n_mid: keep all
    inp = make_inputs(w)
    a = host_arrays(inp)
    dims, prm = dims_of(inp), params_of(w)
    res = oracle.decode(dims, prm, a["q"], a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                        a["block_table"], a["seq_lens"])
    o_s, l_s = oracle.attend(dims, prm, a["q"], a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                             a["block_table"], a["seq_lens"], res["sel_idx"], res["sel_count"], with_lse=True)
    khat, vhat = _pool(inp)
    o_h, l_h = oracle.hca_attend(dims, prm, a["q"], khat, vhat, a["seq_lens"], GROUP)
    out, lse = oracle.lse_merge(o_s, l_s, o_h, l_h)
    G, T = w.num_q_heads // w.num_kv_heads, GROUP * w.block_size
    q = inp["q"].cpu().to(torch.float64)
    scale = 1.0 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        ng = (L + T - 1) // T
        K, V = _tokens(inp, b, "k"), _tokens(inp, b, "v")
        for i in range(w.num_q_heads):
            h = i // G
            keys = torch.cat([K[h], torch.from_numpy(khat[b, :ng, h])])
            vals = torch.cat([V[h], torch.from_numpy(vhat[b, :ng, h])])
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[b, 0, i][None, None, None], keys[None, None], vals[None, None], scale=scale)[0, 0, 0]
            np.testing.assert_allclose(out[b, 0, i], ref.numpy(), rtol=1e-11, atol=1e-12)
            assert lse[b, 0, i] == pytest.approx(float(torch.logsumexp(keys @ q[b, 0, i] * scale, 0)), rel=1e-12)


def test_sparse_branch_lse_is_logsumexp_over_kept_tokens():
    w = SMALL_TOPP
    inp = make_inputs(w)
    a = host_arrays(inp)
    dims, prm = dims_of(inp), params_of(w)
    res = oracle.decode(dims, prm, a["q"], a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                        a["block_table"], a["seq_lens"])
    _, lse = oracle.attend(dims, prm, a["q"], a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                           a["block_table"], a["seq_lens"], res["sel_idx"], res["sel_count"], with_lse=True)
    P, G = w.block_size, w.num_q_heads // w.num_kv_heads
    q = inp["q"].cpu().to(torch.float64)
    K = dequant(inp, "k")
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        for i in range(w.num_q_heads):
            h = i // G
            keep = res["sel_idx"][b, h, :res["sel_count"][b, h]]
            rows = []
            for j in keep:
                page = int(inp["block_table"][b, j])
                rows.append(K[page, h, :min(P, L - int(j) * P)])
            logits = torch.cat(rows) @ q[b, 0, i] / math.sqrt(w.head_dim)
            assert lse[b, 0, i] == pytest.approx(float(torch.logsumexp(logits, 0)), rel=1e-12)
