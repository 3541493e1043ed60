"""Float64 CPU oracle for block-sparse decode attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
has no fallback to it.  The arithmetic lives in ``spattn_oracle.c`` (plain
C, float64); this module only marshals numpy arrays into it.

Every array argument is a numpy array holding the exact stored bytes:
bf16 values as ``uint16`` bit patterns, fp8 e4m3fn values as ``uint8``
codes, scales as ``float32``, tables and lengths as ``int32``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

from . import build as _build

_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "q_tokens", "num_q_heads", "num_kv_heads", "head_dim",
        "block_size", "num_pages", "max_blocks", "max_sel", "kv_fp8")]


class _Params(ctypes.Structure):
    _fields_ = [("sink_blocks", ctypes.c_int), ("local_blocks", ctypes.c_int),
                ("mode", ctypes.c_int), ("top_k", ctypes.c_int),
                ("top_p", ctypes.c_double), ("max_ratio", ctypes.c_double),
                ("sm_scale", ctypes.c_double), ("min_ratio", ctypes.c_double)]


@dataclasses.dataclass
class Dims:
    batch: int
    q_tokens: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_pages: int
    max_blocks: int
    max_sel: int
    kv_fp8: bool = False

    def c(self) -> _Dims:
        return _Dims(self.batch, self.q_tokens, self.num_q_heads, self.num_kv_heads,
                     self.head_dim, self.block_size, self.num_pages, self.max_blocks,
                     self.max_sel, int(self.kv_fp8))


@dataclasses.dataclass
class Params:
    sink_blocks: int = 1
    local_blocks: int = 2
    mode: str = "topk"          # "topk" | "topp" | "topp_anchor"
    top_k: int = 0
    top_p: float = 1.0
    max_ratio: float = 0.0
    sm_scale: float = 0.0
    min_ratio: float = 0.0      # topp_anchor: the cap ratio when the anchors dominate

    def c(self) -> _Params:
        return _Params(self.sink_blocks, self.local_blocks,
                       {"topk": 0, "topp": 1, "topp_anchor": 2}[self.mode], self.top_k,
                       float(self.top_p), float(self.max_ratio), float(self.sm_scale),
                       float(self.min_ratio))


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        for name, args in {
            "spo_compress_keys": [P, P, P, P, P, P],
            "spo_block_scores": [P, P, P, P, P, P, P],
            "spo_select": [P, P, P, P, P, P, P],
            "spo_attend": [P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_int, P, P],
            "spo_hca_pool": [P, P, P, P, P, P, P, ctypes.c_int, P, P],
            "spo_hca_attend": [P, P, P, P, P, P, ctypes.c_int, P, P],
        }.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.spo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.spo_bf16_to_f64.restype = ctypes.c_double
        L.spo_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.spo_e4m3_to_f64.restype = ctypes.c_double
        L.spo_num_threads.restype = ctypes.c_int
        L.spo_set_num_threads.argtypes = [ctypes.c_int]
        L.spo_set_num_threads.restype = None
        L.spo_round_bf16.argtypes = [ctypes.c_double]
        L.spo_round_bf16.restype = ctypes.c_double
        L.spo_round_bf16_array.argtypes = [P, ctypes.c_int64]
        L.spo_round_bf16_array.restype = None
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().spo_num_threads()


def set_num_threads(n: int) -> None:
    """Threads for the following calls (timing of a one-core run)."""
    lib().spo_set_num_threads(n)


def bf16_to_f64(bits: int) -> float:
    return lib().spo_bf16_to_f64(bits)


def e4m3_to_f64(bits: int) -> float:
    return lib().spo_e4m3_to_f64(bits)


def round_bf16(x):
    """The nearest bf16 values (ties to even) of float64 data, as float64:
    the compressed keys of low-precision scoring."""
    if np.isscalar(x):
        return lib().spo_round_bf16(float(x))
    a = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().spo_round_bf16_array(_ptr(a), a.size)
    return a


def _cache_dtype(dims: Dims):
    return np.uint8 if dims.kv_fp8 else np.uint16


def compress_keys(dims: Dims, k_cache, k_scale, block_table, seq_lens) -> np.ndarray:
    """Mean-pooled key of every referenced block: float64 [num_pages][Hkv][d]."""
    kbar = np.zeros((dims.num_pages, dims.num_kv_heads, dims.head_dim), np.float64)
    k_cache = _c(k_cache, _cache_dtype(dims))
    k_scale = _c(k_scale, np.float32) if dims.kv_fp8 else None
    bt, sl = _c(block_table, np.int32), _c(seq_lens, np.int32)
    rc = lib().spo_compress_keys(ctypes.byref(dims.c()), _ptr(k_cache), _ptr(k_scale),
                                 _ptr(bt), _ptr(sl), _ptr(kbar))
    if rc != 0:
        raise ValueError(f"spo_compress_keys failed ({rc})")
    return kbar


def block_scores(dims: Dims, params: Params, q, kbar, block_table, seq_lens) -> np.ndarray:
    """Block scores: float64 [B][Tq][Hkv][max_blocks], -inf outside the middle."""
    s = np.empty((dims.batch, dims.q_tokens, dims.num_kv_heads, dims.max_blocks), np.float64)
    q = _c(q, np.uint16)
    kbar = _c(kbar, np.float64)
    bt, sl = _c(block_table, np.int32), _c(seq_lens, np.int32)
    rc = lib().spo_block_scores(ctypes.byref(dims.c()), ctypes.byref(params.c()), _ptr(q),
                                _ptr(kbar), _ptr(bt), _ptr(sl), _ptr(s))
    if rc != 0:
        raise ValueError(f"spo_block_scores failed ({rc})")
    return s


def select(dims: Dims, params: Params, scores, seq_lens):
    """Kept blocks per (b, h): (sel_idx [B][Hkv][max_sel], sel_count [B][Hkv], margin [B][Hkv])."""
    sel = np.full((dims.batch, dims.num_kv_heads, dims.max_sel), -1, np.int32)
    cnt = np.zeros((dims.batch, dims.num_kv_heads), np.int32)
    margin = np.zeros((dims.batch, dims.num_kv_heads), np.float64)
    scores = _c(scores, np.float64)
    sl = _c(seq_lens, np.int32)
    rc = lib().spo_select(ctypes.byref(dims.c()), ctypes.byref(params.c()), _ptr(scores),
                          _ptr(sl), _ptr(sel), _ptr(cnt), _ptr(margin))
    if rc != 0:
        raise ValueError(f"spo_select failed ({rc}): max_sel too small")
    return sel, cnt, margin


def attend(dims: Dims, params: Params, q, k_cache, v_cache, k_scale, v_scale,
           block_table, seq_lens, sel_idx, sel_count, units=None, with_lse=False):
    """Softmax attention over the kept blocks: float64 [B][Tq][Hq][d]
    (and, with_lse, the ln-sum-exp of each row's logits [B][Tq][Hq]).

    ``units``: optional list of (b, h) pairs to compute; other rows stay 0.
    """
    out = np.zeros((dims.batch, dims.q_tokens, dims.num_q_heads, dims.head_dim), np.float64)
    lse = np.full((dims.batch, dims.q_tokens, dims.num_q_heads), -np.inf) if with_lse else None
    cd = _cache_dtype(dims)
    k_cache, v_cache = _c(k_cache, cd), _c(v_cache, cd)
    ks = _c(k_scale, np.float32) if dims.kv_fp8 else None
    vs = _c(v_scale, np.float32) if dims.kv_fp8 else None
    u = None if units is None else np.ascontiguousarray(np.asarray(units, np.int32).reshape(-1, 2))
    rc = lib().spo_attend(ctypes.byref(dims.c()), ctypes.byref(params.c()), _ptr(_c(q, np.uint16)),
                          _ptr(k_cache), _ptr(v_cache), _ptr(ks), _ptr(vs),
                          _ptr(_c(block_table, np.int32)), _ptr(_c(seq_lens, np.int32)),
                          _ptr(_c(sel_idx, np.int32)), _ptr(_c(sel_count, np.int32)),
                          _ptr(u), 0 if u is None else len(u), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"spo_attend failed ({rc})")
    return (out, lse) if with_lse else out


def hca_pool(dims: Dims, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, group_blocks=2):
    """Mean-pooled K and V of every group of group_blocks logical blocks:
    float64 [B][G_max][Hkv][d] each."""
    gmax = (dims.max_blocks + group_blocks - 1) // group_blocks
    khat = np.zeros((dims.batch, gmax, dims.num_kv_heads, dims.head_dim), np.float64)
    vhat = np.zeros_like(khat)
    cd = _cache_dtype(dims)
    ks = _c(k_scale, np.float32) if dims.kv_fp8 else None
    vs = _c(v_scale, np.float32) if dims.kv_fp8 else None
    rc = lib().spo_hca_pool(ctypes.byref(dims.c()), _ptr(_c(k_cache, cd)), _ptr(_c(v_cache, cd)), _ptr(ks),
                            _ptr(vs), _ptr(_c(block_table, np.int32)), _ptr(_c(seq_lens, np.int32)),
                            group_blocks, _ptr(khat), _ptr(vhat))
    if rc != 0:
        raise ValueError(f"spo_hca_pool failed ({rc})")
    return khat, vhat


def hca_attend(dims: Dims, params: Params, q, khat, vhat, seq_lens, group_blocks=2):
    """Dense attention over the pooled entries: (out [B][Tq][Hq][d], lse [B][Tq][Hq])."""
    out = np.zeros((dims.batch, dims.q_tokens, dims.num_q_heads, dims.head_dim), np.float64)
    lse = np.full((dims.batch, dims.q_tokens, dims.num_q_heads), -np.inf)
    rc = lib().spo_hca_attend(ctypes.byref(dims.c()), ctypes.byref(params.c()), _ptr(_c(q, np.uint16)),
                              _ptr(_c(khat, np.float64)), _ptr(_c(vhat, np.float64)),
                              _ptr(_c(seq_lens, np.int32)), group_blocks, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"spo_hca_attend failed ({rc})")
    return out, lse


def lse_merge(out_a, lse_a, out_b, lse_b):
    """Softmax over the union of two key sets from the two partial results:
    out = (e^lse_a out_a + e^lse_b out_b) / (e^lse_a + e^lse_b), lse = ln of
    the sum (a row with neither keeps 0 and -inf)."""
    m = np.maximum(lse_a, lse_b)
    mm = np.where(np.isfinite(m), m, 0.0)
    wa, wb = np.exp(lse_a - mm), np.exp(lse_b - mm)
    z = wa + wb
    out = (wa[..., None] * out_a + wb[..., None] * out_b) / np.where(z > 0, z, 1.0)[..., None]
    lse = np.where(z > 0, mm + np.log(np.where(z > 0, z, 1.0)), -np.inf)
    return out, lse


def decode(dims: Dims, params: Params, q, k_cache, v_cache, k_scale, v_scale,
           block_table, seq_lens, kbar=None, units=None):
    """The whole path: compress (unless kbar given), score, select, attend.

    Returns a dict with kbar, scores, sel_idx, sel_count, margin, out.
    """
    if kbar is None:
        kbar = compress_keys(dims, k_cache, k_scale, block_table, seq_lens)
    scores = block_scores(dims, params, q, kbar, block_table, seq_lens)
    sel, cnt, margin = select(dims, params, scores, seq_lens)
    out = attend(dims, params, q, k_cache, v_cache, k_scale, v_scale, block_table,
                 seq_lens, sel, cnt, units)
    return dict(kbar=kbar, scores=scores, sel_idx=sel, sel_count=cnt, margin=margin, out=out)


__all__ = ["Dims", "Params", "compress_keys", "block_scores", "select", "attend", "decode",
           "bf16_to_f64", "e4m3_to_f64", "num_threads", "lib"]
