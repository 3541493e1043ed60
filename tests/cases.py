"""Seeded test workloads: small cases the oracle finishes in seconds (several
tiles, ragged tails), plus the five full-size named workloads."""
from block_sparse_kv_spattn_b200.workloads import WORKLOADS, Workload

SMALL_TOPP = Workload("small_topp", batch=2, q_tokens=1, num_q_heads=8, num_kv_heads=2,
                      seq_len=64 * 40 + 17, structure="zipf", mode="topp", top_p=0.9,
                      max_ratio=0.15, seed=11)
SMALL_FP8_CHUNK = Workload("small_fp8_chunk", batch=2, q_tokens=4, num_q_heads=8, num_kv_heads=2,
                           seq_len=64 * 30 + 5, kv_fp8=True, structure="zipf", mode="topk",
                           max_ratio=0.12, seed=12)
SMALL_RAGGED = Workload("small_ragged", batch=3, q_tokens=1, num_q_heads=4, num_kv_heads=1,
                        seq_len=0, ragged=(100, 5000), structure="planted", n_planted=3,
                        mode="topk", top_k=5, seed=13)
# one case per attention row-group shape (rows = Tq * Hq / Hkv = 8, 16, 64, 8)
GQA8_TOPP = Workload("gqa8_topp", batch=3, q_tokens=1, num_q_heads=64, num_kv_heads=8,
                     seq_len=64 * 300 + 31, structure="zipf", mode="topp", top_p=0.95,
                     max_ratio=0.20, seed=14)
MQA16_TOPK = Workload("mqa16_topk", batch=2, q_tokens=1, num_q_heads=16, num_kv_heads=1,
                      seq_len=64 * 500 + 1, structure="planted", n_planted=30, mode="topk",
                      max_ratio=0.10, seed=15)
CHUNK16_FP8 = Workload("chunk16_fp8", batch=2, q_tokens=16, num_q_heads=32, num_kv_heads=8,
                       seq_len=64 * 200 + 3, kv_fp8=True, structure="zipf", mode="topk",
                       max_ratio=0.12, seed=16)
CHUNK2_TOPP = Workload("chunk2_topp", batch=2, q_tokens=2, num_q_heads=8, num_kv_heads=2,
                       seq_len=64 * 50 + 63, structure="zipf", mode="topp", top_p=0.9,
                       max_ratio=0.15, seed=17)
GQA4_128K_SMALL = WORKLOADS["decode_128k_b2"]
# anchor-adaptive cap (ratio 10-20 % of the middle blocks)
SMALL_ANCHOR = Workload("small_anchor", batch=3, q_tokens=1, num_q_heads=8, num_kv_heads=2,
                        seq_len=64 * 120 + 9, structure="zipf", mode="topp_anchor", top_p=0.9,
                        min_ratio=0.10, max_ratio=0.20, seed=18)
CHUNK2_ANCHOR = Workload("chunk2_anchor", batch=2, q_tokens=2, num_q_heads=16, num_kv_heads=4,
                         seq_len=64 * 90 + 40, structure="planted", n_planted=8, mode="topp_anchor",
                         top_p=0.8, min_ratio=0.05, max_ratio=0.25, seed=19)

# bf16 cache with 64 query rows per KV head (8 tokens x 8 heads): the
# many-row tensor-core kernel
CHUNK8_WIDE = Workload("chunk8_wide", batch=2, q_tokens=8, num_q_heads=16, num_kv_heads=2,
                       seq_len=64 * 70 + 21, structure="zipf", mode="topp", top_p=0.9,
                       max_ratio=0.2, seed=20)

SMALL_CASES = [WORKLOADS["tiny_4k_gqa4"], SMALL_TOPP, SMALL_FP8_CHUNK, SMALL_RAGGED, GQA8_TOPP,
               MQA16_TOPK, CHUNK16_FP8, CHUNK2_TOPP, GQA4_128K_SMALL, SMALL_ANCHOR, CHUNK2_ANCHOR, CHUNK8_WIDE]
