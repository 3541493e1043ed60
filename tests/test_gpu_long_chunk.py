"""Prefill chunks with more than 64 query rows per KV head, against the oracle.

A (request, KV head) with Tq * group query rows runs as one attention unit
per 64-row tile, each over the same kept blocks with its own causal mask;
the scoring grid tiles the chunk's tokens; the selection is the union of the
tokens' own selections.
Every step is compared element by element with the float64 oracle, whose
causal mask over a chunk longer than the local window is pinned on the CPU
(tests/test_oracle_pins.py).
"""
import pytest

from block_sparse_kv_spattn_b200.workloads import Workload, make_inputs
from tests.parity import compare, run_library

pytestmark = pytest.mark.gpu

# 40 tokens x group 4 = 160 rows (3 tiles, the last partial), bf16, top-k
LONG_BF16 = Workload("long_bf16", batch=2, q_tokens=40, num_q_heads=8, num_kv_heads=2,
                     seq_len=64 * 40 + 9, structure="zipf", mode="topk", max_ratio=0.3, seed=41)
# 24 tokens x group 4 = 96 rows over an fp8 cache
LONG_FP8 = Workload("long_fp8", batch=2, q_tokens=24, num_q_heads=32, num_kv_heads=8,
                    seq_len=64 * 60 + 33, kv_fp8=True, structure="zipf", mode="topk", max_ratio=0.12, seed=42)
# a 200-token chunk (longer than the two local blocks), MQA group 4: 800 rows, top-p
LONG_TOPP = Workload("long_topp", batch=1, q_tokens=200, num_q_heads=4, num_kv_heads=1,
                     seq_len=64 * 30 + 1, structure="zipf", mode="topp", top_p=0.9, max_ratio=0.3, seed=43)
# 64 tokens x group 8 = 512 rows per KV head (8 full tiles), bf16 and fp8
ROWS512_BF16 = Workload("rows512_bf16", batch=2, q_tokens=64, num_q_heads=16, num_kv_heads=2,
                        seq_len=64 * 48 + 20, structure="zipf", mode="topk", max_ratio=0.2, seed=44)
ROWS512_FP8 = Workload("rows512_fp8", batch=1, q_tokens=64, num_q_heads=32, num_kv_heads=4,
                       seq_len=64 * 36 + 63, kv_fp8=True, structure="zipf", mode="topp", top_p=0.95,
                       max_ratio=0.25, seed=45)

CASES = [LONG_BF16, LONG_FP8, LONG_TOPP, ROWS512_BF16, ROWS512_FP8]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_long_chunk_parity(cuda, w):
    inp = make_inputs(w, device="cuda")
    gpu = run_library(inp)
    s = compare(inp, gpu)
    assert s["exact_rows"] + s["replayed_rows"] == w.batch * w.num_kv_heads
