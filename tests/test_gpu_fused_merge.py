"""The merge inside the attention kernel: repeated calls on one
workspace give identical results (the arrival counts clear themselves), one
workspace serves calls of different dims, units with nothing kept get zero
rows and -inf log-sum-exp, and the fused and separate-merge shapes agree with
the oracle (the parity suite covers that)."""
import pytest
import torch

from block_sparse_kv_spattn_b200 import spattn
from block_sparse_kv_spattn_b200.workloads import WORKLOADS, make_inputs
from tests.parity import lib_params

pytestmark = pytest.mark.gpu


def _selection(inp, params):
    w = inp["workload"]
    q, kc, bt, sl = inp["q"], inp["k_cache"], inp["block_table"], inp["seq_lens"]
    kbar = torch.empty((kc.shape[0], kc.shape[1], 128), device="cuda")
    spattn.compress_keys(kc, inp["k_scale"], bt, sl, kbar, num_q_heads=w.num_q_heads)
    dims = spattn.dims_for(q, kc, bt)
    max_sel = spattn.required_max_sel(dims, params)
    scores = torch.empty((w.batch, w.q_tokens, w.num_kv_heads, bt.shape[1]), device="cuda")
    sel_idx = torch.empty((w.batch, w.num_kv_heads, max_sel), dtype=torch.int32, device="cuda")
    sel_count = torch.empty((w.batch, w.num_kv_heads), dtype=torch.int32, device="cuda")
    spattn.block_scores(q, kbar, bt, sl, scores, params, k_cache=kc)
    spattn.select(scores, sl, sel_idx, sel_count, params, q=q, k_cache=kc, block_table=bt)
    return sel_idx, sel_count


@pytest.mark.parametrize("name", ["decode_128k_b2", "ragged_b32", "tiny_4k_gqa4"])
def test_repeated_calls_identical(cuda, name):
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    params = lib_params(w)
    sel_idx, sel_count = _selection(inp, params)
    args = (inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
            inp["block_table"], inp["seq_lens"], sel_idx, sel_count)
    dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], sel_idx.shape[-1])
    ws = spattn.alloc_workspace(dims, params, "cuda")
    outs = []
    for _ in range(3):
        out = torch.full(tuple(inp["q"].shape), float("nan"), device="cuda")
        spattn.decode_selected(*args, out, ws, params)
        assert spattn.device_status() == 0
        outs.append(out)
    assert torch.isfinite(outs[0]).all()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_one_workspace_for_two_shapes(cuda):
    big, small = WORKLOADS["decode_128k_b2"], WORKLOADS["ragged_b32"]
    res = {}
    wss = {}
    for w in (big, small):
        inp = make_inputs(w, device="cuda")
        params = lib_params(w)
        sel_idx, sel_count = _selection(inp, params)
        dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], sel_idx.shape[-1])
        wss[w.name] = spattn.workspace_size(dims, params)
        res[w.name] = (inp, params, sel_idx, sel_count)
    ws = torch.empty(max(wss.values()), dtype=torch.uint8, device="cuda")
    spattn.workspace_init(ws)
    for name in (big.name, small.name, big.name):
        inp, params, sel_idx, sel_count = res[name]
        args = (inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
                inp["block_table"], inp["seq_lens"], sel_idx, sel_count)
        ref_ws = spattn.alloc_workspace(
            spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], sel_idx.shape[-1]), params, "cuda")
        ref = torch.empty(tuple(inp["q"].shape), device="cuda")
        spattn.decode_selected(*args, ref, ref_ws, params)
        out = torch.empty(tuple(inp["q"].shape), device="cuda")
        spattn.decode_selected(*args, out, ws, params)
        assert spattn.device_status() == 0
        assert torch.equal(out, ref), name


def test_empty_units_zero_rows_and_lse(cuda):
    w = WORKLOADS["decode_128k_b2"]
    inp = make_inputs(w, device="cuda")
    params = lib_params(w)
    sel_idx, sel_count = _selection(inp, params)
    sel_count[0, 1] = 0
    sel_count[1, 5] = 0
    args = (inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
            inp["block_table"], inp["seq_lens"], sel_idx, sel_count)
    dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], sel_idx.shape[-1])
    ws = spattn.alloc_workspace(dims, params, "cuda")
    out = torch.full(tuple(inp["q"].shape), float("nan"), device="cuda")
    lse = torch.full(tuple(inp["q"].shape[:3]), float("nan"), device="cuda")
    spattn.decode_selected(*args, out, ws, params, lse=lse)
    assert spattn.device_status() == 0
    G = w.num_q_heads // w.num_kv_heads
    for b, h in ((0, 1), (1, 5)):
        assert torch.all(out[b, :, h * G:(h + 1) * G] == 0)
        assert torch.all(lse[b, :, h * G:(h + 1) * G] == float("-inf"))
    assert torch.isfinite(out).all()
