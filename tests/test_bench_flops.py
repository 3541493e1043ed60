"""bench.py's host-side accounting: the algorithmic FLOP count of the sparse
attention against a brute-force count of (query row, visible kept token)
pairs on small cases (decode rows see every kept token; chunk rows are
causal within the chunk; partly filled last block), and the oracle sample
both host legs time, with its scale to a whole step."""
import random

import torch

import bench
from block_sparse_kv_spattn_b200.workloads import Workload


def _brute(w, lens, sel_idx, sel_count):
    P, G, Tq = w.block_size, w.num_q_heads // w.num_kv_heads, w.q_tokens
    pairs = 0
    for b, L in enumerate(lens):
        for h in range(w.num_kv_heads):
            kept = set(sel_idx[b][h][:sel_count[b][h]])
            for t in range(Tq):
                me = L - Tq + t
                for pos in range(L):
                    if pos // P in kept and pos <= me:
                        pairs += G
    return pairs * 4 * w.head_dim


def _case(seed, q_tokens, lens, hq=8, hkv=2):
    rng = random.Random(seed)
    w = Workload("t", batch=len(lens), q_tokens=q_tokens, num_q_heads=hq, num_kv_heads=hkv, seq_len=max(lens))
    max_sel = 12
    sel_idx, sel_count = [], []
    for L in lens:
        nb = (L + w.block_size - 1) // w.block_size
        rows_i, rows_c = [], []
        for _ in range(hkv):
            k = rng.randint(0, min(max_sel, nb))
            ids = sorted(rng.sample(range(nb), k))
            rows_i.append(ids + [0] * (max_sel - k))
            rows_c.append(k)
        sel_idx.append(rows_i)
        sel_count.append(rows_c)
    inp = {"workload": w, "seq_lens": torch.tensor(lens, dtype=torch.int32)}
    got = bench.attention_flops(inp, torch.tensor(sel_idx, dtype=torch.int32), torch.tensor(sel_count, dtype=torch.int32))
    assert got == _brute(w, lens, sel_idx, sel_count)
    return got


def test_decode_rows_see_every_kept_token():
    assert _case(1, 1, [64 * 9, 64 * 5 + 17]) > 0


def test_chunk_rows_are_causal():
    _case(2, 40, [64 * 6 + 5, 64 * 3 + 40])
    _case(3, 7, [64 * 2 + 63, 64 * 4])


def test_empty_selection_has_no_flops():
    w = Workload("t", batch=1, q_tokens=3, num_q_heads=4, num_kv_heads=1, seq_len=256)
    inp = {"workload": w, "seq_lens": torch.tensor([256], dtype=torch.int32)}
    assert bench.attention_flops(inp, torch.zeros((1, 1, 4), dtype=torch.int32),
                                 torch.zeros((1, 1), dtype=torch.int32)) == 0


def test_oracle_sample_of_the_last_chunk_tokens():
    """The CPU baseline's smallest sample (the last n query tokens of one KV
    head) runs the oracle over the whole chunk's selection."""
    from block_sparse_kv_spattn_b200.workloads import make_inputs
    w = Workload("t", batch=1, q_tokens=8, num_q_heads=8, num_kv_heads=2, seq_len=64 * 12 + 5, structure="zipf",
                 mode="topk", max_ratio=0.3, seed=5)
    inp = make_inputs(w, device="cpu")
    full = bench.oracle_request(inp, 0, heads=[0])()
    part = bench.oracle_request(inp, 0, heads=[0], last_tokens=3)()
    assert full == part > 0


def test_oracle_sample_scaling(monkeypatch):
    """The host legs' sample and its scale to the step: the whole request
    when it is short, one KV head when the request is long, the last few
    query tokens of one head when even that is long."""
    from block_sparse_kv_spattn_b200.workloads import make_inputs
    w = Workload("t", batch=3, q_tokens=8, num_q_heads=8, num_kv_heads=2, seq_len=64 * 6, structure="zipf",
                 mode="topk", max_ratio=0.3, seed=6)
    inp = make_inputs(w, device="cpu")
    for t_tok, kind, scale, kept_scale in ((0.1, "request 0", 3, 3), (1.0, "KV head 0", 6, 6),
                                           (4.0, "last 2 of 8", 24, 6)):
        monkeypatch.setattr(bench, "_time_runs", lambda run, seconds, min_runs=1, max_runs=None, t=t_tok: [t])
        smp = bench.oracle_sample(inp)
        assert kind in smp["what"], smp["what"]
        assert smp["scale"] == scale and smp["kept_scale"] == kept_scale
        assert smp["run"]() > 0
