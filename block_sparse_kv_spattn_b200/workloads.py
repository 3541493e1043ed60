"""Seeded synthetic workloads for block-sparse decode attention.

This module only draws inputs: it holds none of the attention method's
arithmetic (no pooling, scoring, selection or softmax).  Both the CUDA path
and the CPU oracle consume exactly the bytes it produces.

Shapes follow the configuration table of "Claude Opus 长上下文 KV Cache 稀疏注意力"
(§可落地的配置参数与监控要点: 64-token blocks, 1 sink block, 2 local blocks,
10-20 % retention) and the five named workloads below.

Recipe (all configurations):
  * q, K, V ~ N(0, 1), rounded to bf16 (round-to-nearest-even).
  * u[b, h] = unit vector along the sum of the query rows of KV-head group h
    at the last query token; "boosted" blocks get coef * sqrt(d) * u added to
    every key of the block before rounding.
  * planted:  n_planted distinct middle blocks per (b, h) get coef 0.5.
  * zipf:     a random permutation gives every middle block a rank r >= 1;
              coef = 1.0 * r ** -1.1 (power-law block importance).
  * pages: one page per (request, block); page ids are a seeded random
    permutation (identity for the contiguous tiny case).  Unused block-table
    columns hold -1.  Token slots past the end of a request's last block hold
    NaN, so any read of them shows up in the result.
  * fp8 caches: per (page, KV head) scale = amax(|x|) / 448 over the filled
    tokens (1 when amax is 0); code = e4m3fn(x / scale), round to nearest
    even; K and V are scaled separately.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BLOCK = 64
HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_tokens: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: int                      # fixed context (ignored when ragged)
    ragged: Optional[tuple] = None    # (lo, hi): log-uniform lengths, rounded to 64
    kv_fp8: bool = False
    structure: str = "zipf"           # "zipf" | "planted" | "none"
    n_planted: int = 0
    contiguous: bool = False
    mode: str = "topp"                # "topk" | "topp" | "topp_anchor"
    top_k: int = 0
    top_p: float = 1.0
    max_ratio: float = 0.0
    min_ratio: float = 0.0            # topp_anchor: the cap ratio when the anchors dominate
    kbar_bf16: bool = False           # compressed keys stored as bf16 (low-precision scoring)
    hca: bool = False                 # add the dense branch over 128-token mean entries
    sink_blocks: int = 1
    local_blocks: int = 2
    head_dim: int = HEAD_DIM
    block_size: int = BLOCK
    seed: int = 1234

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 1 request, 8 q heads / 2 KV heads, 4096 tokens, contiguous pages,
    # 6 planted middle blocks per KV head, top-k 8.
    "tiny_4k_gqa4": Workload("tiny_4k_gqa4", batch=1, q_tokens=1, num_q_heads=8, num_kv_heads=2,
                             seq_len=4096, structure="planted", n_planted=6, contiguous=True,
                             mode="topk", top_k=8, seed=1235),
    # 8 requests x 128K tokens, 32 q heads / 8 KV heads, power-law block
    # importance, top-p 0.9 capped at 15 % of the middle blocks.
    "decode_128k_b8": Workload("decode_128k_b8", batch=8, q_tokens=1, num_q_heads=32, num_kv_heads=8,
                               seq_len=131072, structure="zipf", mode="topp", top_p=0.9,
                               max_ratio=0.15, seed=1236),
    # the gate shape with the anchor-adaptive cap: ratio between 10 % and 20 %
    # of the middle blocks by how far the best middle block stands above the
    # sink and local blocks
    "decode_128k_b8_anchor": Workload("decode_128k_b8_anchor", batch=8, q_tokens=1, num_q_heads=32,
                                      num_kv_heads=8, seq_len=131072, structure="zipf",
                                      mode="topp_anchor", top_p=0.9, min_ratio=0.10, max_ratio=0.20,
                                      seed=1241),
    # the gate shape scored from bf16 compressed keys (half the scoring bytes)
    "decode_128k_b8_kbar16": Workload("decode_128k_b8_kbar16", batch=8, q_tokens=1, num_q_heads=32,
                                      num_kv_heads=8, seq_len=131072, structure="zipf", mode="topp",
                                      top_p=0.9, max_ratio=0.15, kbar_bf16=True, seed=1236),
    # the gate shape with the weight-free HCA branch beside the sparse one
    # (pooled 128-token entries, dense attention, log-sum-exp merge)
    "decode_128k_b8_hca": Workload("decode_128k_b8_hca", batch=8, q_tokens=1, num_q_heads=32,
                                   num_kv_heads=8, seq_len=131072, structure="zipf", mode="topp",
                                   top_p=0.9, max_ratio=0.15, hca=True, seed=1236),
    # the same shape with 2 requests: small enough for detailed profiling
    "decode_128k_b2": Workload("decode_128k_b2", batch=2, q_tokens=1, num_q_heads=32, num_kv_heads=8,
                               seq_len=131072, structure="zipf", mode="topp", top_p=0.9,
                               max_ratio=0.15, seed=1240),
    # ... and with the HCA branch (profiling size of decode_128k_b8_hca)
    "decode_128k_b2_hca": Workload("decode_128k_b2_hca", batch=2, q_tokens=1, num_q_heads=32, num_kv_heads=8,
                                   seq_len=131072, structure="zipf", mode="topp", top_p=0.9,
                                   max_ratio=0.15, hca=True, seed=1240),
    # 32 requests, lengths log-uniform in [8K, 256K], 64 q heads / 8 KV heads,
    # top-p 0.95 capped at 20 %.
    "ragged_b32": Workload("ragged_b32", batch=32, q_tokens=1, num_q_heads=64, num_kv_heads=8,
                           seq_len=0, ragged=(8192, 262144), structure="zipf", mode="topp",
                           top_p=0.95, max_ratio=0.20, seed=1237),
    # 2 requests x 1M tokens, 16 q heads / 1 KV head, 1000 needle blocks,
    # top-k 10 % of the middle blocks.
    "decode_1m_mqa": Workload("decode_1m_mqa", batch=2, q_tokens=1, num_q_heads=16, num_kv_heads=1,
                              seq_len=1048576, structure="planted", n_planted=1000, mode="topk",
                              max_ratio=0.10, seed=1238),
    # 4 requests x 512K tokens, 16-token query chunks sharing one union
    # selection, fp8 e4m3 cache with per-(page, head) scales, top-k 12 %.
    "chunk16_fp8_512k": Workload("chunk16_fp8_512k", batch=4, q_tokens=16, num_q_heads=32,
                                 num_kv_heads=8, seq_len=524288, kv_fp8=True, structure="zipf",
                                 mode="topk", max_ratio=0.12, seed=1239),
    # the fp8 chunk shape at 128K context: small enough for detailed profiling
    "chunk16_fp8_128k": Workload("chunk16_fp8_128k", batch=4, q_tokens=16, num_q_heads=32,
                                 num_kv_heads=8, seq_len=131072, kv_fp8=True, structure="zipf",
                                 mode="topk", max_ratio=0.12, seed=1242),
    # a prefill chunk: 64 tokens x 8 query heads per KV head = 512 query rows
    # per (request, KV head), eight 64-row tiles over the chunk's union
    # selection (top-k 10 % per token), bf16 cache
    "prefill_chunk64_128k": Workload("prefill_chunk64_128k", batch=2, q_tokens=64, num_q_heads=64,
                                     num_kv_heads=8, seq_len=131072, structure="zipf", mode="topk",
                                     max_ratio=0.10, seed=1243),
}

BENCH_WORKLOAD = "decode_128k_b8"


def seq_lens_for(w: Workload, gen: torch.Generator) -> torch.Tensor:
    if w.ragged is None:
        return torch.full((w.batch,), w.seq_len, dtype=torch.int32)
    lo, hi = w.ragged
    u = torch.rand(w.batch, generator=gen, dtype=torch.float64, device=gen.device).cpu()
    lens = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    lens = (torch.round(lens / w.block_size) * w.block_size).clamp(min=w.block_size)
    return lens.to(torch.int32)


def _quant_e4m3(x: torch.Tensor, filled: torch.Tensor):
    """x: float32 [n, Hkv, P, d] (slots past `filled` tokens are ignored)."""
    P = x.shape[2]
    mask = (torch.arange(P, device=x.device)[None, :] < filled[:, None])  # [n, P]
    ax = (x.abs() * mask[:, None, :, None]).amax(dim=(2, 3))              # [n, Hkv]
    scale = torch.where(ax > 0, ax / 448.0, torch.ones_like(ax))
    y = (x / scale[:, :, None, None]).clamp(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


@torch.no_grad()
def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw one workload on `device`.  Returns a dict of tensors and metadata.

    q        bf16  [B][Tq][Hq][d]
    k_cache  bf16  [num_pages][Hkv][P][d]   (uint8 e4m3fn codes when kv_fp8)
    v_cache  same as k_cache
    k_scale  f32   [num_pages][Hkv]         (ones for bf16 caches)
    v_scale  f32   [num_pages][Hkv]
    block_table int32 [B][max_blocks]       (-1 past a request's last block)
    seq_lens int32 [B]
    boosted  list per b of int64 [Hkv][n] middle block ids that got an offset
             (planted ids, or the Zipf rank order, best first)
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    P, D, H, Hq, Tq = w.block_size, w.head_dim, w.num_kv_heads, w.num_q_heads, w.q_tokens
    G = Hq // H
    seq_lens = seq_lens_for(w, gen)
    nbs = [(int(L) + P - 1) // P for L in seq_lens]
    num_pages = sum(nbs)
    max_blocks = max(nbs)
    if w.contiguous:
        perm = torch.arange(num_pages, dtype=torch.int64)
    else:
        perm = torch.randperm(num_pages, generator=gen, device=device).cpu()
    block_table = torch.full((w.batch, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b, nb in enumerate(nbs):
        block_table[b, :nb] = perm[off:off + nb].to(torch.int32)
        off += nb

    q = torch.randn((w.batch, Tq, Hq, D), generator=gen, device=device).to(torch.bfloat16)
    cdt = torch.uint8 if w.kv_fp8 else torch.bfloat16
    k_cache = torch.empty((num_pages, H, P, D), dtype=cdt, device=device)
    v_cache = torch.empty((num_pages, H, P, D), dtype=cdt, device=device)
    k_scale = torch.ones((num_pages, H), dtype=torch.float32, device=device)
    v_scale = torch.ones((num_pages, H), dtype=torch.float32, device=device)
    boosted = []
    sqrt_d = math.sqrt(D)
    bt_dev = block_table.to(device=device, dtype=torch.int64)
    for b, nb in enumerate(nbs):
        L = int(seq_lens[b])
        S, W = w.sink_blocks, w.local_blocks
        n_mid = max(0, nb - S - W)
        u = q[b, Tq - 1].float().view(H, G, D).sum(dim=1)
        u = u / u.norm(dim=-1, keepdim=True).clamp_min(1e-30)            # [H, D]
        coef = torch.zeros((H, nb), dtype=torch.float32, device=device)
        ids = torch.zeros((H, 0), dtype=torch.int64)
        if n_mid > 0 and w.structure == "planted":
            n = min(w.n_planted, n_mid)
            ids = torch.stack([torch.randperm(n_mid, generator=gen, device=device)[:n] + S
                               for _ in range(H)]).cpu()
            coef.scatter_(1, ids.to(device), 0.5)
        elif n_mid > 0 and w.structure == "zipf":
            order = torch.stack([torch.randperm(n_mid, generator=gen, device=device) + S
                                 for _ in range(H)])                       # rank r-1 -> block
            ranks = torch.arange(1, n_mid + 1, device=device, dtype=torch.float32)
            coef.scatter_(1, order, ranks.pow(-1.1).expand(H, n_mid).contiguous())
            ids = order.cpu()
        boosted.append(ids)
        filled = torch.clamp(L - torch.arange(nb, device=device) * P, max=P)   # [nb]
        tail = torch.arange(P, device=device)[None, :] >= filled[:, None]      # [nb, P]
        pages = bt_dev[b, :nb]
        for which, cache, scale_out in ((0, k_cache, k_scale), (1, v_cache, v_scale)):
            x = torch.randn((nb, H, P, D), generator=gen, device=device)
            if which == 0:
                x += (coef.t()[:, :, None, None] * sqrt_d) * u[None, :, None, :]
            x = x.to(torch.bfloat16).float()
            if w.kv_fp8:
                codes, sc = _quant_e4m3(x, filled)
                codes[tail[:, None, :, None].expand_as(codes)] = 0x7F        # e4m3fn NaN
                cache[pages] = codes
                scale_out[pages] = sc
            else:
                x[tail[:, None, :, None].expand_as(x)] = float("nan")
                cache[pages] = x.to(torch.bfloat16)
    return dict(workload=w, q=q, k_cache=k_cache, v_cache=v_cache, k_scale=k_scale,
                v_scale=v_scale, block_table=block_table.to(device), seq_lens=seq_lens.to(device),
                boosted=boosted, num_pages=num_pages, max_blocks=max_blocks)
