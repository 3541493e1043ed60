"""Run the CUDA library and the float64 oracle on the same bytes and compare.

Tolerances (derived in the design notes from fp32 arithmetic):
  kbar    |gpu - oracle| <= 2e-6 * max|column| + 1e-7 * |oracle|; bf16 compressed
          keys: the oracle's mean rounded to bf16, within one bf16 step
          (2^-7 |oracle|) on top of that, and the scores checked against the
          oracle's scoring of the GPU's own compressed keys
  scores  |gpu - oracle| <= 1e-5 * max(1, |oracle|)
  indices bit-exact where the oracle's decision margin exceeds 1e-4;
          otherwise replayed: the oracle's selection run on the GPU's own
          fp32 scores must give the GPU's indices (top-p cuts that land within
          the fp32 rounding band of p may take either neighbour)
  out     max |gpu - oracle| <= 2e-3 (bf16 KV), 2e-2 (fp8 KV), the oracle
          attending over the GPU's selection
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_kv_spattn_b200 import spattn
from oracle.marshal import bits16, cache_bytes, dims_of, params_of, subproblem

MARGIN = 1e-4
TOPP_BAND = 1e-5
OUT_TOL = {False: 2e-3, True: 2e-2}


def lib_params(w) -> spattn.Params:
    return spattn.Params(sink_blocks=w.sink_blocks, local_blocks=w.local_blocks, mode=w.mode,
                         top_k=w.top_k, top_p=w.top_p, max_ratio=w.max_ratio, min_ratio=w.min_ratio)


def run_library(inp: dict, params: spattn.Params | None = None, kbar_bf16: bool = False) -> dict:
    """compress (all blocks) + decode through the C ABI; results on device."""
    w = inp["workload"]
    params = params or lib_params(w)
    q, kc, vc = inp["q"], inp["k_cache"], inp["v_cache"]
    bt, sl = inp["block_table"], inp["seq_lens"]
    dev = q.device
    kbar = torch.full((kc.shape[0], kc.shape[1], kc.shape[3]), float("nan"), device=dev,
                      dtype=torch.bfloat16 if kbar_bf16 else torch.float32)
    spattn.compress_keys(kc, inp["k_scale"], bt, sl, kbar, num_q_heads=w.num_q_heads,
                         q_tokens=w.q_tokens)
    dims = spattn.dims_for(q, kc, bt)
    max_sel = spattn.required_max_sel(dims, params)
    B, Hkv = w.batch, w.num_kv_heads
    sel_idx = torch.full((B, Hkv, max_sel), -1, dtype=torch.int32, device=dev)
    sel_count = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
    scores = torch.empty((B, w.q_tokens, Hkv, bt.shape[1]), dtype=torch.float32, device=dev)
    out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device=dev)
    dims.max_sel = max_sel
    ws = spattn.alloc_workspace(dims, params, dev)
    spattn.decode(q, kc, vc, inp["k_scale"], inp["v_scale"], bt, sl, kbar, out, sel_idx, sel_count,
                  ws, params, scores_out=scores)
    status = spattn.device_status()
    return dict(kbar=kbar, scores=scores, sel_idx=sel_idx, sel_count=sel_count, out=out,
                status=status, max_sel=max_sel)


def anchor_cap(w, row_scores: np.ndarray, S: int, nb: int) -> int:
    """The anchor-adaptive cap of one score row, computed as the library does
    (double arithmetic on the fp32 scores and parameters)."""
    W = w.local_blocks
    mid = row_scores[S:nb - W].astype(np.float64)
    a = max([float(row_scores[j]) for j in list(range(S)) + list(range(nb - W, nb))], default=-math.inf)
    hi, lo = float(mid.max()), float(mid.min())
    r = (hi - a) / (hi - lo) if hi > lo else 0.0
    r = min(max(r, 0.0), 1.0)
    mn, mx = float(np.float32(w.min_ratio)), float(np.float32(w.max_ratio))
    return min(len(mid), math.floor((mn + r * (mx - mn)) * len(mid)))


def _topp_prefix_ok(w, row_scores: np.ndarray, S: int, nb: int, got_mid: list[int]) -> bool:
    """GPU top-p set is the ranked prefix of its own scores of a length that
    sits within the fp32 rounding band of p (or at the cap)."""
    mid = np.arange(S, max(S, nb - w.local_blocks))
    s = row_scores[mid].astype(np.float64)
    order = sorted(range(len(mid)), key=lambda i: (-s[i], i))
    m = len(got_mid)
    if sorted(mid[order[:m]].tolist()) != sorted(got_mid):
        return False
    e = np.exp(s[order] - s[order[0]])
    c = np.cumsum(e / e.sum())
    if w.mode == "topp_anchor":
        k_max = anchor_cap(w, row_scores, S, nb)
    else:
        k_max = math.floor(w.max_ratio * len(mid)) if w.max_ratio > 0 else len(mid)
    if m == k_max:
        return True
    near = [abs(c[i] - w.top_p) for i in (m - 2, m - 1) if 0 <= i < len(c)]
    return bool(near) and min(near) < TOPP_BAND


def compare(inp: dict, gpu: dict, requests=None, params_override=None, kbar_bf16: bool = False,
            attend_requests=None) -> dict:
    """Compare every step for the listed requests (default: all); the
    attention only for ``attend_requests`` (default: the same requests).
    Returns a summary (max errors, exact/replayed row counts); raises
    AssertionError on any violation."""
    w = inp["workload"]
    fp8 = w.kv_fp8
    requests = range(w.batch) if requests is None else requests
    attend_requests = set(requests if attend_requests is None else attend_requests)
    summary = dict(kbar_err=0.0, score_err=0.0, out_err=0.0, exact_rows=0, replayed_rows=0)
    assert gpu["status"] == 0, f"device status word {gpu['status']:#x}"
    opar = params_of(w, **(params_override or {}))
    H, G, P = w.num_kv_heads, w.num_q_heads // w.num_kv_heads, w.block_size
    for b in requests:
        sub = subproblem(inp, b)
        L = int(inp["seq_lens"][b])
        nb = (L + P - 1) // P
        dims = dims_of(sub, max_sel=gpu["max_sel"])
        qh, kh, vh = bits16(sub["q"]), cache_bytes(sub["k_cache"]), cache_bytes(sub["v_cache"])
        ksc, vsc = sub["k_scale"].cpu().numpy(), sub["v_scale"].cpu().numpy()
        bt, sl = sub["block_table"].cpu().numpy(), sub["seq_lens"].cpu().numpy()
        # 1. compressed keys
        kb_o = oracle.compress_keys(dims, kh, ksc, bt, sl)
        pages = sub["page_of_block"][:nb]
        kb_g = gpu["kbar"][pages].double().cpu().numpy()
        if nb:
            K = (sub["k_cache"][:nb].view(torch.float8_e4m3fn).double() * sub["k_scale"][:nb, :, None, None].double()
                 if fp8 else sub["k_cache"][:nb].double())
            filled = torch.clamp(L - torch.arange(nb, device=K.device) * P, max=P)
            tmask = (torch.arange(P, device=K.device)[None, :] < filled[:, None])[:, None, :, None]
            colmax = torch.where(tmask, K.abs(), torch.zeros_like(K)).amax(dim=2).cpu().numpy()
            if kbar_bf16:
                kb_o = oracle.round_bf16(kb_o)
                tol = 2e-6 * colmax + 2.0 ** -7 * np.abs(kb_o[:nb]) + 1e-30
            else:
                tol = 2e-6 * colmax + 1e-7 * np.abs(kb_o[:nb])
            err = np.abs(kb_g - kb_o[:nb])
            assert np.all(err <= tol), f"kbar b={b}: max err {err.max():.3g}"
            summary["kbar_err"] = max(summary["kbar_err"], float(err.max()))
        # 2. scores
        sc_o = oracle.block_scores(dims, opar, qh, kb_o, bt, sl)
        sc_g = gpu["scores"][b:b + 1].double().cpu().numpy()
        # the scoring itself: against the oracle's scores of the GPU's own keys
        sc_c = oracle.block_scores(dims, opar, qh, kb_g, bt, sl) if kbar_bf16 and nb else sc_o
        fin = np.isfinite(sc_o)
        assert np.array_equal(fin, np.isfinite(sc_g)), f"scores b={b}: -inf pattern differs"
        if fin.any():
            err = np.abs(sc_g[fin] - sc_c[fin])
            assert np.all(err <= 1e-5 * np.maximum(1.0, np.abs(sc_c[fin]))), \
                f"scores b={b}: max err {err.max():.3g}"
            summary["score_err"] = max(summary["score_err"], float(err.max()))
        # 3. selection: exact where the margin is clear, else replay
        sel_o, cnt_o, margin = oracle.select(dims, opar, sc_o, sl)
        sel_r, cnt_r, _ = oracle.select(dims, opar, sc_g, sl)
        g_idx = gpu["sel_idx"][b].cpu().numpy()
        g_cnt = gpu["sel_count"][b].cpu().numpy()
        for h in range(H):
            got = g_idx[h, :g_cnt[h]].tolist()
            if margin[0, h] > MARGIN:
                assert got == sel_o[0, h, :cnt_o[0, h]].tolist(), f"selection b={b} h={h} (margin {margin[0, h]:.3g})"
                summary["exact_rows"] += 1
            else:
                want = sel_r[0, h, :cnt_r[0, h]].tolist()
                if got != want:
                    assert w.mode in ("topp", "topp_anchor") and w.q_tokens == 1, f"replay b={b} h={h} differs"
                    keep = set(range(min(w.sink_blocks, nb))) | set(range(max(0, nb - w.local_blocks), nb))
                    got_mid = [j for j in got if j not in keep]
                    assert _topp_prefix_ok(w, sc_g[0, 0, h], w.sink_blocks, nb, got_mid), \
                        f"replay b={b} h={h}: not a valid top-p cut"
                summary["replayed_rows"] += 1
        # 4. attention over the GPU's own selection
        if b not in attend_requests:
            continue
        summary["attended"] = summary.get("attended", 0) + 1
        sel_g = np.full((1, H, gpu["max_sel"]), -1, np.int32)
        sel_g[0] = g_idx
        out_o = oracle.attend(dims, opar, qh, kh, vh, ksc, vsc, bt, sl, sel_g, g_cnt[None])
        out_g = gpu["out"][b:b + 1].double().cpu().numpy()
        assert np.all(np.isfinite(out_g)), f"out b={b} has non-finite values"
        err = np.abs(out_g - out_o)
        assert err.max() <= OUT_TOL[fp8], f"out b={b}: max err {err.max():.3g}"
        summary["out_err"] = max(summary["out_err"], float(err.max()))
    return summary
