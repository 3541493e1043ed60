"""Hand workload tensors to the float64 oracle as the exact stored bytes.

Marshalling only (bit patterns, sizes, parameters, one request's pages
gathered in logical order); none of the method's arithmetic.  Like the rest
of this package it is test infrastructure: the tests, the smoke check and the
benchmark's CPU-baseline and reference legs use it; the CUDA library never
does.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cache_bytes(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.uint8:
        return t.detach().contiguous().cpu().numpy()
    return bits16(t)


def dims_of(inp: dict, max_sel: int | None = None) -> oracle.Dims:
    w = inp["workload"]
    return oracle.Dims(batch=w.batch, q_tokens=w.q_tokens, num_q_heads=w.num_q_heads,
                       num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                       block_size=w.block_size, num_pages=inp["num_pages"],
                       max_blocks=inp["max_blocks"],
                       max_sel=inp["max_blocks"] if max_sel is None else max_sel,
                       kv_fp8=w.kv_fp8)


def params_of(w, **kw) -> oracle.Params:
    """The oracle's parameters as the library receives them: the fp32 values
    of the float fields (so a ratio gives the same floor on both sides)."""
    f32 = lambda x: float(np.float32(x))
    p = oracle.Params(sink_blocks=w.sink_blocks, local_blocks=w.local_blocks, mode=w.mode,
                      top_k=w.top_k, top_p=f32(w.top_p), max_ratio=f32(w.max_ratio),
                      min_ratio=f32(w.min_ratio))
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def host_arrays(inp: dict) -> dict:
    return dict(q=bits16(inp["q"]), k_cache=cache_bytes(inp["k_cache"]),
                v_cache=cache_bytes(inp["v_cache"]),
                k_scale=inp["k_scale"].cpu().numpy(), v_scale=inp["v_scale"].cpu().numpy(),
                block_table=inp["block_table"].cpu().numpy(),
                seq_lens=inp["seq_lens"].cpu().numpy())


def dequant(inp: dict, which: str) -> torch.Tensor:
    """float64 [num_pages][Hkv][P][d] through torch's own dtype conversions."""
    c = inp[which + "_cache"].cpu()
    if c.dtype == torch.uint8:
        x = c.view(torch.float8_e4m3fn).to(torch.float64)
        return x * inp[which + "_scale"].cpu().to(torch.float64)[:, :, None, None]
    return c.to(torch.float64)


def run_oracle(inp: dict, params=None, units=None, max_sel=None) -> dict:
    w = inp["workload"]
    a = host_arrays(inp)
    return oracle.decode(dims_of(inp, max_sel), params or params_of(w), a["q"], a["k_cache"],
                         a["v_cache"], a["k_scale"], a["v_scale"], a["block_table"],
                         a["seq_lens"], units=units)


def subproblem(inp: dict, b: int) -> dict:
    """Request b alone, its pages gathered in logical order (page id = block id)."""
    w = inp["workload"]
    L = int(inp["seq_lens"][b])
    P = w.block_size
    nb = max(1, (L + P - 1) // P)
    pages = inp["block_table"][b, :nb].long().clamp_min(0)
    sub = dict(inp)
    sub["workload"] = w.replace(batch=1)
    sub["q"] = inp["q"][b:b + 1]
    sub["k_cache"] = inp["k_cache"][pages].contiguous()
    sub["v_cache"] = inp["v_cache"][pages].contiguous()
    sub["k_scale"] = inp["k_scale"][pages].contiguous()
    sub["v_scale"] = inp["v_scale"][pages].contiguous()
    bt = torch.full((1, inp["max_blocks"]), -1, dtype=torch.int32, device=inp["q"].device)
    bt[0, :nb] = torch.arange(nb, dtype=torch.int32, device=bt.device)
    sub["block_table"] = bt
    sub["seq_lens"] = inp["seq_lens"][b:b + 1]
    sub["num_pages"] = nb
    sub["page_of_block"] = pages
    return sub
