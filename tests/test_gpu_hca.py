"""The HCA branch on the GPU against the float64 oracle.

"CSA + HCA 混合注意力机制" §5.1-5.2 (pooled 128-token entries, dense attention over
them) and §6 (the two branches joined by their log-sum-exp).  Tolerances,
from the fp32 arithmetic of the kernels:
  khat / vhat   fp32 sums of at most 128 terms: |gpu - oracle| <= 128 u mean|x|
                with u = 2^-24, bounded here by 2e-5 (1 + |oracle|) (|x| <~ 10)
  hca out, lse  fp32 logits of d = 128 products and exp2 of the hardware:
                1e-4 (outputs are convex combinations of |v| <~ 10 values)
  sparse lse    the attention's fp32 maxima and sums: 1e-3 absolute
  merged out    the sparse branch's bound: 2e-3 (bf16 KV), 2e-2 (fp8 KV)
The oracle always takes what the GPU took as its input where the branch
under test starts (the GPU's selection, the GPU's pooled entries), so each
check measures one step.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_kv_spattn_b200 import spattn
from block_sparse_kv_spattn_b200.workloads import WORKLOADS, Workload, make_inputs
from tests.cases import CHUNK2_TOPP, CHUNK16_FP8, GQA8_TOPP, MQA16_TOPK, SMALL_FP8_CHUNK, SMALL_RAGGED, SMALL_TOPP
from oracle.marshal import dims_of, host_arrays, params_of
from tests.parity import OUT_TOL, lib_params, run_library

pytestmark = pytest.mark.gpu

GROUP = spattn.HCA_BLOCKS
POOL_TOL, HCA_TOL, LSE_TOL = 2e-5, 1e-4, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda):
    spattn.load()
    spattn.device_status()


def gpu_pool(inp):
    kc, bt = inp["k_cache"], inp["block_table"]
    G = spattn.hca_entries(bt)
    shape = (bt.shape[0], kc.shape[1], G, kc.shape[3])    # [B][Hkv][G][d]
    khat = torch.full(shape, float("nan"), device="cuda")
    vhat = torch.full(shape, float("nan"), device="cuda")
    spattn.hca_pool(kc, inp["v_cache"], inp["k_scale"], inp["v_scale"], bt, inp["seq_lens"], khat, vhat)
    return khat, vhat


def gpu_hca_attend(inp, khat, vhat):
    w, q = inp["workload"], inp["q"]
    out = torch.full(tuple(q.shape), float("nan"), device="cuda")
    lse = torch.full(tuple(q.shape[:3]), float("nan"), device="cuda")
    spattn.hca_attend(q, khat, vhat, inp["seq_lens"], out, lse, lib_params(w), k_cache=inp["k_cache"],
                      block_table=inp["block_table"])
    return out, lse


def oracle_pool(inp):
    a = host_arrays(inp)
    return oracle.hca_pool(dims_of(inp), a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                           a["block_table"], a["seq_lens"], GROUP)


def host(t):
    """GPU entries [B][Hkv][G][d] -> the oracle's [B][G][Hkv][d], float64."""
    return t.permute(0, 2, 1, 3).double().cpu().numpy()


def _max_err(gpu, ref):
    g = gpu.double().cpu().numpy() if torch.is_tensor(gpu) else gpu
    both_inf = np.isinf(g) & np.isinf(ref) & (np.sign(g) == np.sign(ref))
    with np.errstate(invalid="ignore"):
        d = np.where(both_inf, 0.0, np.abs(g - ref))
    return float(np.nan_to_num(d, nan=np.inf).max()) if d.size else 0.0


HCA_CASES = [SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED, GQA8_TOPP, CHUNK2_TOPP, MQA16_TOPK, CHUNK16_FP8]


@pytest.mark.parametrize("w", HCA_CASES, ids=lambda w: w.name)
def test_hca_pool_parity(w):
    inp = make_inputs(w, device="cuda")
    khat, vhat = gpu_pool(inp)
    assert spattn.device_status() == 0
    rk, rv = oracle_pool(inp)
    for g, r in ((khat, rk), (vhat, rv)):
        err = np.abs(host(g) - r) / (1.0 + np.abs(r))
        assert err.max() <= POOL_TOL


@pytest.mark.parametrize("w", HCA_CASES, ids=lambda w: w.name)
def test_hca_attend_parity(w):
    inp = make_inputs(w, device="cuda")
    khat, vhat = gpu_pool(inp)
    out, lse = gpu_hca_attend(inp, khat, vhat)
    assert spattn.device_status() == 0
    a = host_arrays(inp)
    ro, rl = oracle.hca_attend(dims_of(inp), params_of(w), a["q"], host(khat),
                               host(vhat), a["seq_lens"], GROUP)
    assert _max_err(out, ro) <= HCA_TOL
    assert _max_err(lse, rl) <= HCA_TOL * (1 + np.abs(np.nan_to_num(rl, neginf=0)).max())
    assert torch.equal(torch.isinf(lse).cpu(), torch.from_numpy(np.isinf(rl)))


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, GQA8_TOPP, CHUNK2_TOPP], ids=lambda w: w.name)
def test_sparse_branch_lse(w):
    """spattn_decode_selected_lse: the row's log-sum-exp over the kept tokens
    (the output itself equals spattn_decode_selected's)."""
    inp = make_inputs(w, device="cuda")
    gpu = run_library(inp)
    params = lib_params(w)
    dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], gpu["max_sel"])
    ws = spattn.alloc_workspace(dims, params, "cuda")
    out = torch.empty_like(gpu["out"])
    lse = torch.full(tuple(inp["q"].shape[:3]), float("nan"), device="cuda")
    spattn.decode_selected(inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
                           inp["block_table"], inp["seq_lens"], gpu["sel_idx"], gpu["sel_count"], out, ws,
                           params, lse=lse)
    assert spattn.device_status() == 0
    assert torch.equal(out, gpu["out"])
    a = host_arrays(inp)
    ro, rl = oracle.attend(dims_of(inp, gpu["max_sel"]), params_of(w), a["q"], a["k_cache"], a["v_cache"],
                           a["k_scale"], a["v_scale"], a["block_table"], a["seq_lens"],
                           gpu["sel_idx"].cpu().numpy(), gpu["sel_count"].cpu().numpy(), with_lse=True)
    assert _max_err(lse, rl) <= LSE_TOL
    assert _max_err(out, ro) <= OUT_TOL[w.kv_fp8]


def test_lse_merge_parity_and_in_place():
    g = torch.Generator(device="cuda").manual_seed(31)
    B, Tq, Hq = 3, 2, 8
    oa = torch.randn((B, Tq, Hq, 128), generator=g, device="cuda")
    ob = torch.randn((B, Tq, Hq, 128), generator=g, device="cuda")
    la = torch.randn((B, Tq, Hq), generator=g, device="cuda") * 30
    lb = torch.randn((B, Tq, Hq), generator=g, device="cuda") * 30
    la[0, 0, :3] = -float("inf")          # one side empty
    lb[0, 1, :2] = -float("inf")
    la[1, 0, 0] = lb[1, 0, 0] = -float("inf")   # both empty
    oa[0, 0, :3] = 0
    ob[0, 1, :2] = 0
    oa[1, 0, 0] = ob[1, 0, 0] = 0
    ro, rl = oracle.lse_merge(oa.double().cpu().numpy(), la.double().cpu().numpy(),
                              ob.double().cpu().numpy(), lb.double().cpu().numpy())
    out = torch.empty_like(oa)
    lse = torch.empty_like(la)
    spattn.lse_merge(oa, la, ob, lb, out, lse)
    torch.cuda.synchronize()
    assert _max_err(out, ro) <= 1e-5
    assert _max_err(lse, rl) <= 1e-5
    assert torch.all(out[1, 0, 0] == 0) and lse[1, 0, 0] == -float("inf")
    # in place over the first input
    spattn.lse_merge(oa, la, ob, lb, oa, la)
    torch.cuda.synchronize()
    assert torch.equal(oa, out) and torch.equal(la, lse)


def hybrid_gpu(inp):
    """Sparse branch with lse + HCA branch + log-sum-exp merge, all on the GPU."""
    w = inp["workload"]
    gpu = run_library(inp)
    params = lib_params(w)
    dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], gpu["max_sel"])
    ws = spattn.alloc_workspace(dims, params, "cuda")
    o_s = torch.empty_like(gpu["out"])
    l_s = torch.empty(tuple(inp["q"].shape[:3]), device="cuda")
    spattn.decode_selected(inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
                           inp["block_table"], inp["seq_lens"], gpu["sel_idx"], gpu["sel_count"], o_s, ws,
                           params, lse=l_s)
    khat, vhat = gpu_pool(inp)
    o_h, l_h = gpu_hca_attend(inp, khat, vhat)
    out, lse = torch.empty_like(o_s), torch.empty_like(l_s)
    spattn.lse_merge(o_s, l_s, o_h, l_h, out, lse)
    assert spattn.device_status() == 0
    return gpu, khat, vhat, out, lse


def test_hca_attend_merge_is_attend_then_lse_merge():
    """spattn_hca_attend_merge against the oracle's merge of the oracle's
    two branches (GPU selection and entries as inputs), and against the
    GPU's own two-launch composition."""
    for w in (SMALL_TOPP, CHUNK2_TOPP, GQA8_TOPP):
        inp = make_inputs(w, device="cuda")
        gpu, khat, vhat, out2, lse2 = hybrid_gpu(inp)
        params = lib_params(w)
        dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], gpu["max_sel"])
        ws = spattn.alloc_workspace(dims, params, "cuda")
        o_s = torch.empty_like(gpu["out"])
        l_s = torch.empty(tuple(inp["q"].shape[:3]), device="cuda")
        spattn.decode_selected(inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
                               inp["block_table"], inp["seq_lens"], gpu["sel_idx"], gpu["sel_count"], o_s, ws,
                               params, lse=l_s)
        out = torch.full_like(o_s, float("nan"))
        lse = torch.full_like(l_s, float("nan"))
        spattn.hca_attend(inp["q"], khat, vhat, inp["seq_lens"], out, lse, params, k_cache=inp["k_cache"],
                          block_table=inp["block_table"], merge_with=(o_s, l_s))
        assert spattn.device_status() == 0
        ro, rl = hybrid_oracle(inp, gpu, khat, vhat)
        assert _max_err(out, ro) <= OUT_TOL[w.kv_fp8]
        assert _max_err(lse, rl) <= LSE_TOL
        assert _max_err(out, out2.double().cpu().numpy()) <= 1e-5


def hybrid_oracle(inp, gpu, khat, vhat, requests=None):
    """The oracle's sparse branch over the GPU's selection and its HCA branch
    over the GPU's pooled entries, merged by the oracle."""
    w = inp["workload"]
    a = host_arrays(inp)
    dims, prm = dims_of(inp, gpu["max_sel"]), params_of(w)
    units = None if requests is None else [(b, h) for b in requests for h in range(w.num_kv_heads)]
    o_s, l_s = oracle.attend(dims, prm, a["q"], a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"],
                             a["block_table"], a["seq_lens"], gpu["sel_idx"].cpu().numpy(),
                             gpu["sel_count"].cpu().numpy(), units=units, with_lse=True)
    o_h, l_h = oracle.hca_attend(dims, prm, a["q"], host(khat), host(vhat),
                                 a["seq_lens"], GROUP)
    return oracle.lse_merge(o_s, l_s, o_h, l_h)


@pytest.mark.parametrize("w", [SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED, CHUNK2_TOPP], ids=lambda w: w.name)
def test_hybrid_step_parity(w):
    inp = make_inputs(w, device="cuda")
    gpu, khat, vhat, out, lse = hybrid_gpu(inp)
    ro, rl = hybrid_oracle(inp, gpu, khat, vhat)
    assert _max_err(out, ro) <= OUT_TOL[w.kv_fp8]
    assert _max_err(lse, rl) <= LSE_TOL


def test_hybrid_full_size_sampled():
    """decode_128k_b8 (the benchmark's workload) through the hybrid path;
    requests 0 and 7 through the oracle, every pooled entry checked."""
    w = WORKLOADS["decode_128k_b8"]
    inp = make_inputs(w, device="cuda")
    gpu, khat, vhat, out, lse = hybrid_gpu(inp)
    rk, rv = oracle_pool(inp)
    assert (np.abs(host(khat) - rk) / (1 + np.abs(rk))).max() <= POOL_TOL
    assert (np.abs(host(vhat) - rv) / (1 + np.abs(rv))).max() <= POOL_TOL
    reqs = [0, 7]
    ro, rl = hybrid_oracle(inp, gpu, khat, vhat, requests=reqs)
    assert _max_err(out[reqs], ro[reqs]) <= OUT_TOL[False]
    assert _max_err(lse[reqs], rl[reqs]) <= LSE_TOL


def test_hca_edge_lengths():
    """Empty request, one token, 127 / 128 / 129 tokens (entry boundary), and
    a chunk of 4 query tokens whose last entry is visible to the last token
    only."""
    w = Workload("hca_edges", batch=6, q_tokens=4, num_q_heads=8, num_kv_heads=2, seq_len=64 * 8,
                 structure="zipf", mode="topk", top_k=2, seed=24)
    inp = make_inputs(w, device="cuda")
    inp["seq_lens"] = torch.tensor([0, 1, 127, 128, 129, 64 * 8], dtype=torch.int32, device="cuda")
    khat, vhat = gpu_pool(inp)
    out, lse = gpu_hca_attend(inp, khat, vhat)
    assert spattn.device_status() == 0
    rk, rv = oracle_pool(inp)
    assert (np.abs(host(khat) - rk) / (1 + np.abs(rk))).max() <= POOL_TOL
    a = host_arrays(inp)
    ro, rl = oracle.hca_attend(dims_of(inp), params_of(w), a["q"], host(khat),
                               host(vhat), a["seq_lens"], GROUP)
    assert _max_err(out, ro) <= HCA_TOL
    assert torch.equal(torch.isinf(lse).cpu(), torch.from_numpy(np.isinf(rl)))
    # request 0 sees nothing; request 1 (one token): only its last query
    # token sees entry 0; request 4 (129 tokens): query tokens at 125, 126
    # see nothing, 127 sees entry 0, 128 sees entries 0 and 1
    assert torch.all(out[0] == 0) and torch.all(lse[0] == -float("inf"))
    assert torch.all(torch.isinf(lse[1, :3])) and torch.all(torch.isfinite(lse[1, 3]))
    assert torch.all(torch.isinf(lse[4, :2])) and torch.all(torch.isfinite(lse[4, 2:]))


def test_incremental_pool_matches_full():
    """Appending tokens and pooling only the touched entries gives the same
    entries as pooling everything."""
    w = WORKLOADS["tiny_4k_gqa4"].replace(seq_len=64 * 22)
    inp = make_inputs(w, device="cuda")
    kc, vc, bt = inp["k_cache"], inp["v_cache"], inp["block_table"]
    old = torch.tensor([64 * 20 + 10], dtype=torch.int32, device="cuda")
    new = old + 60
    G = spattn.hca_entries(bt)
    shape = (1, kc.shape[1], G, 128)
    inc = torch.zeros(shape, device="cuda")
    inc_v = torch.zeros(shape, device="cuda")
    spattn.hca_pool(kc, vc, inp["k_scale"], inp["v_scale"], bt, old, inc, inc_v)
    g = torch.Generator(device="cuda").manual_seed(6)
    for cache in (kc, vc):
        for tok in range(int(old[0]), int(new[0])):
            cache[int(bt[0, tok // 64]), :, tok % 64] = torch.randn((cache.shape[1], 128), generator=g,
                                                                   device="cuda").to(cache.dtype)
    spattn.hca_pool(kc, vc, inp["k_scale"], inp["v_scale"], bt, new, inc, inc_v, old_lens=old, q_tokens=60)
    full = torch.zeros(shape, device="cuda")
    full_v = torch.zeros(shape, device="cuda")
    spattn.hca_pool(kc, vc, inp["k_scale"], inp["v_scale"], bt, new, full, full_v)
    assert spattn.device_status() == 0
    torch.testing.assert_close(inc, full, rtol=0, atol=0)
    torch.testing.assert_close(inc_v, full_v, rtol=0, atol=0)
