"""spattn_decode_selected_noalloc against spattn_decode_selected.

Some callers cannot allocate device memory where they call the attention:
an engine plugin whose host owns every allocation, code inside a CUDA stream
capture, or a latency-bound serving loop that must not allocate or free.
For them the library has an entry point that takes no workspace and keeps its
split-KV partials in a fixed scratch array built into the library.  This test
calls it through the C ABI several times in a row, on two shapes in turn,
and checks each output against the workspace entry point's output on the
same selection: the two must be identical.  The file is named so that pytest collects it
last; it also passes alone in a fresh process.
"""
import ctypes

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


def _case(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    params = lib_params(w)
    sel_idx, sel_count = _selection(inp, params)
    args = (inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"],
            inp["block_table"], inp["seq_lens"], sel_idx, sel_count)
    ref = torch.empty(tuple(inp["q"].shape), device="cuda")
    dims = spattn.dims_for(inp["q"], inp["k_cache"], inp["block_table"], sel_idx.shape[-1])
    ws = spattn.alloc_workspace(dims, params, "cuda")
    spattn.decode_selected(*args, ref, ws, params)
    return inp, params, args, ref


def test_noalloc_matches_workspace_entry_point(cuda):
    """Calls alternate between a small and a large shape (tiny, 128K, tiny,
    128K), so a call that read partial results left in the shared
    scratch by the call before it would differ from the workspace entry
    point.  Both entry points run the same kernels with the same split on the
    same selection, so the outputs must be identical bit for bit."""
    cases = {name: _case(name) for name in ("tiny_4k_gqa4", "decode_128k_b2")}
    for call, name in enumerate(("tiny_4k_gqa4", "decode_128k_b2", "tiny_4k_gqa4", "decode_128k_b2")):
        inp, params, args, ref = cases[name]
        out = torch.full(tuple(inp["q"].shape), float("nan"), device="cuda")
        spattn.decode_selected_noalloc(*args, out, params)
        assert spattn.device_status() == 0
        assert torch.isfinite(out).all(), f"call {call} ({name})"
        err = (out - ref).abs().max().item()
        assert torch.equal(out, ref), f"call {call} ({name}): max |noalloc - workspace| = {err:.3g}"


def test_noalloc_rejects_dims_beyond_its_scratch(cuda):
    """64 query rows per KV head over 128 requests x 8 KV heads need far more
    than the built-in scratch: refused on the host, nothing enqueued."""
    lib = spattn.load()
    d = spattn.CDims(128, 16, 32, 8, 128, 64, 1000, 100, 100, 0, 0)
    p = spattn.Params(top_k=4).c()
    dummy = ctypes.c_void_p(256)
    st = lib.spattn_decode_selected_noalloc(ctypes.byref(d), ctypes.byref(p), dummy, dummy, dummy,
                                            None, None, dummy, dummy, dummy, dummy, dummy, None)
    assert st == 2
    assert b"scratch" in lib.spattn_last_error()
