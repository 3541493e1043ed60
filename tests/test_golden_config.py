"""The page's printed configuration table, checked against the oracle.

Fixture: tests/golden/config_table.txt (values as printed in the configuration
table of "Claude Opus 长上下文 KV Cache 稀疏注意力", section
可落地的配置参数与监控要点).
"""
import math
import os

import numpy as np
import pytest

import oracle
from block_sparse_kv_spattn_b200.workloads import WORKLOADS

HERE = os.path.dirname(os.path.abspath(__file__))


def _table():
    out = {}
    with open(os.path.join(HERE, "golden", "config_table.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (x.strip() for x in line.split("="))
                out[k] = float(v)
    return out


T = _table()


def test_workloads_use_the_printed_block_sink_and_local_sizes():
    for w in WORKLOADS.values():
        assert w.block_size == T["block_size_tokens"]
        assert w.sink_blocks == T["sink_blocks"]
        assert w.local_blocks == T["local_blocks"]
        assert w.sink_blocks * w.block_size == T["sink_tokens"]
        assert w.local_blocks * w.block_size == T["local_tokens"]


@pytest.mark.parametrize("ratio", [T["sparsity_ratio_min"], T["sparsity_ratio_max"]])
def test_always_kept_tokens_and_ratio(ratio):
    """Under the printed parameters the first 64 and the last 128 tokens are
    always kept, whatever the scores, and the middle keeps floor(ratio * n)."""
    P, S, W = int(T["block_size_tokens"]), int(T["sink_blocks"]), int(T["local_blocks"])
    nb = 200
    n_mid = nb - S - W
    dims = oracle.Dims(batch=1, q_tokens=1, num_q_heads=1, num_kv_heads=1, head_dim=128,
                       block_size=P, num_pages=nb, max_blocks=nb, max_sel=nb)
    rng = np.random.default_rng(7)
    s = np.full((1, 1, 1, nb), -np.inf)
    s[0, 0, 0, S:nb - W] = -100.0 - rng.random(n_mid)     # middle scores all very low
    prm = oracle.Params(sink_blocks=S, local_blocks=W, mode="topk", top_k=0, max_ratio=ratio)
    sel, cnt, _ = oracle.select(dims, prm, s, np.array([nb * P], np.int32))
    kept = sel[0, 0, :cnt[0, 0]]
    tokens = {int(j) * P + t for j in kept for t in range(P)}
    assert set(range(int(T["sink_tokens"]))) <= tokens
    assert set(range(nb * P - int(T["local_tokens"]), nb * P)) <= tokens
    assert cnt[0, 0] - S - W == math.floor(ratio * n_mid)
