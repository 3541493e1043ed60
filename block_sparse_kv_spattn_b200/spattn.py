"""ctypes binding of libspattn (include/spattn.h): argument marshalling only.

Every function takes torch CUDA tensors, derives the C structs from their
shapes, and calls the entry point of the same name on the current CUDA
stream (or the one given).  All arithmetic happens in the library's kernels;
if the library is missing this module raises instead of computing anything
else.

Layouts are those of the header: q bf16 [B][Tq][Hq][128]; caches bf16 (or
uint8 e4m3fn codes) [num_pages][Hkv][64][128]; scales f32 [num_pages][Hkv];
block_table int32 [B][max_blocks]; seq_lens int32 [B]; kbar f32
[num_pages][Hkv][128]; scores f32 [B][Tq][Hkv][max_blocks]; sel_idx int32
[B][Hkv][max_sel]; sel_count int32 [B][Hkv]; out f32 [B][Tq][Hq][128];
lse f32 [B][Tq][Hq]; khat / vhat f32 [B][Hkv][ceil(max_blocks / 2)][128].
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libspattn.so")

SPATTN_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "WORKSPACE",
                5: "TIMEOUT", 6: "DEVICE"}
DEV_BAD_PAGE, DEV_BAD_BLOCK, DEV_SEL_OVERFLOW, DEV_WAIT_TIMEOUT, DEV_BAD_LEN = 1, 2, 4, 8, 16
KV_BF16, KV_FP8_E4M3 = 0, 1
SEL_TOPK, SEL_TOPP, SEL_TOPP_ANCHOR = 0, 1, 2
SEL_MODES = {"topk": SEL_TOPK, "topp": SEL_TOPP, "topp_anchor": SEL_TOPP_ANCHOR}
KBAR_F32, KBAR_BF16 = 0, 1

EXPORTS = ("spattn_required_max_sel", "spattn_compress_keys", "spattn_block_scores",
           "spattn_select", "spattn_decode_workspace_size", "spattn_decode_selected",
           "spattn_decode", "spattn_last_error", "spattn_get_device_status", "spattn_version",
           "spattn_decode_selected_noalloc", "spattn_decode_selected_lse", "spattn_hca_entries",
           "spattn_hca_pool", "spattn_hca_attend", "spattn_lse_merge", "spattn_hca_attend_merge",
           "spattn_hca_workspace_size")


class SpattnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"spattn {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class CDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "q_tokens", "num_q_heads", "num_kv_heads", "head_dim", "block_size",
        "num_pages", "max_blocks_per_seq", "max_sel", "kv_dtype", "kbar_dtype")]


class CParams(ctypes.Structure):
    _fields_ = [("sink_blocks", ctypes.c_int32), ("local_blocks", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float),
                ("max_ratio", ctypes.c_float), ("sm_scale", ctypes.c_float), ("min_ratio", ctypes.c_float)]


@dataclasses.dataclass
class Params:
    """Selection parameters (spattn_params)."""
    sink_blocks: int = 1
    local_blocks: int = 2
    mode: str = "topk"      # "topk" | "topp" | "topp_anchor"
    top_k: int = 0
    top_p: float = 1.0
    max_ratio: float = 0.0
    sm_scale: float = 0.0
    min_ratio: float = 0.0  # topp_anchor: the cap ratio when the anchors dominate

    def c(self) -> CParams:
        return CParams(self.sink_blocks, self.local_blocks, SEL_MODES[self.mode],
                       self.top_k, self.top_p, self.max_ratio, self.sm_scale, self.min_ratio)


_lib = None


def load() -> ctypes.CDLL:
    """Load libspattn.so from the package directory (build it with
    ``python -m block_sparse_kv_spattn_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_kv_spattn_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    sig = {
        "spattn_required_max_sel": ([P, P], I32),
        "spattn_compress_keys": ([P, P, P, P, P, P, P, P], ctypes.c_int),
        "spattn_block_scores": ([P, P, P, P, P, P, P, P], ctypes.c_int),
        "spattn_select": ([P, P, P, P, P, P, P], ctypes.c_int),
        "spattn_decode_workspace_size": ([P, P], ctypes.c_size_t),
        "spattn_decode_selected": ([P] * 13 + [ctypes.c_size_t, P], ctypes.c_int),
        "spattn_decode": ([P] * 15 + [ctypes.c_size_t, P], ctypes.c_int),
        "spattn_last_error": ([], ctypes.c_char_p),
        "spattn_get_device_status": ([P, P], ctypes.c_int),
        "spattn_version": ([], ctypes.c_char_p),
        "spattn_decode_selected_noalloc": ([P] * 13, ctypes.c_int),
        "spattn_decode_selected_lse": ([P] * 14 + [ctypes.c_size_t, P], ctypes.c_int),
        "spattn_hca_entries": ([P], I32),
        "spattn_hca_pool": ([P] * 11, ctypes.c_int),
        "spattn_hca_attend": ([P] * 8 + [P, ctypes.c_size_t, P], ctypes.c_int),
        "spattn_hca_workspace_size": ([P], ctypes.c_size_t),
        "spattn_lse_merge": ([P] * 8, ctypes.c_int),
        "spattn_hca_attend_merge": ([P] * 10 + [P, ctypes.c_size_t, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(status: int):
    if status != SPATTN_OK:
        raise SpattnError(status, load().spattn_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("spattn takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("spattn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def kbar_dtype_of(kbar) -> int:
    """fp32 compressed keys, or bf16 (low-precision scoring)."""
    return KBAR_BF16 if kbar is not None and kbar.dtype == torch.bfloat16 else KBAR_F32


def dims_for(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
             max_sel: int = 0, kbar=None) -> CDims:
    B, Tq, Hq, D = q.shape
    num_pages, Hkv, P, D2 = k_cache.shape
    kv = KV_FP8_E4M3 if k_cache.dtype in (torch.uint8, torch.float8_e4m3fn) else KV_BF16
    return CDims(B, Tq, Hq, Hkv, D, P, num_pages, block_table.shape[1], max_sel, kv, kbar_dtype_of(kbar))


def required_max_sel(dims: CDims, params: Params) -> int:
    n = load().spattn_required_max_sel(ctypes.byref(dims), ctypes.byref(params.c()))
    if n < 0:
        raise SpattnError(1, load().spattn_last_error().decode() or "invalid dims or params")
    return n


def workspace_size(dims: CDims, params: Params) -> int:
    n = load().spattn_decode_workspace_size(ctypes.byref(dims), ctypes.byref(params.c()))
    if n == 0:
        raise SpattnError(1, "invalid dims or params")
    return n


def alloc_workspace(dims: CDims, params: Params, device) -> torch.Tensor:
    return torch.empty(workspace_size(dims, params), dtype=torch.uint8, device=device)


def compress_keys(k_cache, k_scale, block_table, seq_lens, kbar, old_lens=None, *,
                  num_q_heads: int = 1, q_tokens: int = 1, stream=None):
    num_pages, Hkv, P, D = k_cache.shape
    kv = KV_FP8_E4M3 if k_cache.dtype in (torch.uint8, torch.float8_e4m3fn) else KV_BF16
    dims = CDims(seq_lens.shape[0], q_tokens, max(num_q_heads, Hkv), Hkv, D, P, num_pages,
                 block_table.shape[1], 0, kv, kbar_dtype_of(kbar))
    _check(load().spattn_compress_keys(ctypes.byref(dims), _p(k_cache),
                                       _p(k_scale) if kv == KV_FP8_E4M3 else None,
                                       _p(block_table), _p(old_lens), _p(seq_lens), _p(kbar),
                                       _stream(stream)))


def block_scores(q, kbar, block_table, seq_lens, scores, params: Params, *, k_cache, stream=None):
    dims = dims_for(q, k_cache, block_table, kbar=kbar)
    _check(load().spattn_block_scores(ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(kbar),
                                      _p(block_table), _p(seq_lens), _p(scores), _stream(stream)))


def select(scores, seq_lens, sel_idx, sel_count, params: Params, *, q, k_cache, block_table,
           stream=None):
    dims = dims_for(q, k_cache, block_table, sel_idx.shape[-1])
    _check(load().spattn_select(ctypes.byref(dims), ctypes.byref(params.c()), _p(scores),
                                _p(seq_lens), _p(sel_idx), _p(sel_count), _stream(stream)))


def decode_selected(q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, sel_idx,
                    sel_count, out, workspace, params: Params, stream=None, lse=None):
    """Attention over the given selection; with ``lse`` (f32 [B][Tq][Hq])
    also each row's log-sum-exp (spattn_decode_selected_lse)."""
    dims = dims_for(q, k_cache, block_table, sel_idx.shape[-1])
    fp8 = dims.kv_dtype == KV_FP8_E4M3
    args = [ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(k_cache), _p(v_cache),
            _p(k_scale) if fp8 else None, _p(v_scale) if fp8 else None, _p(block_table),
            _p(seq_lens), _p(sel_idx), _p(sel_count), _p(out)]
    tail = [_p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)]
    if lse is None:
        _check(load().spattn_decode_selected(*args, *tail))
    else:
        _check(load().spattn_decode_selected_lse(*args, _p(lse), *tail))


def decode_selected_noalloc(q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, sel_idx,
                            sel_count, out, params: Params, stream=None):
    """decode_selected with the library's built-in scratch instead of a
    workspace: for callers that cannot allocate device memory at the call."""
    dims = dims_for(q, k_cache, block_table, sel_idx.shape[-1])
    fp8 = dims.kv_dtype == KV_FP8_E4M3
    _check(load().spattn_decode_selected_noalloc(
        ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(k_cache), _p(v_cache),
        _p(k_scale) if fp8 else None, _p(v_scale) if fp8 else None, _p(block_table),
        _p(seq_lens), _p(sel_idx), _p(sel_count), _p(out), _stream(stream)))


def decode(q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, kbar, out, sel_idx,
           sel_count, workspace, params: Params, scores_out=None, stream=None):
    dims = dims_for(q, k_cache, block_table, sel_idx.shape[-1], kbar=kbar)
    fp8 = dims.kv_dtype == KV_FP8_E4M3
    _check(load().spattn_decode(
        ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(k_cache), _p(v_cache),
        _p(k_scale) if fp8 else None, _p(v_scale) if fp8 else None, _p(block_table),
        _p(seq_lens), _p(kbar), _p(out), _p(sel_idx), _p(sel_count), _p(scores_out),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


# ------------------------------------------------------------------ HCA branch

HCA_BLOCKS = 2      # blocks per pooled entry (128 tokens)


def hca_entries(block_table) -> int:
    """Entries per request of the khat / vhat buffers."""
    return (block_table.shape[1] + HCA_BLOCKS - 1) // HCA_BLOCKS


def hca_pool(k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, khat, vhat, old_lens=None, *,
             q_tokens: int = 1, stream=None):
    """Mean K and V of every 128-token entry: khat / vhat f32 [B][Hkv][G][128]."""
    num_pages, Hkv, P, D = k_cache.shape
    kv = KV_FP8_E4M3 if k_cache.dtype in (torch.uint8, torch.float8_e4m3fn) else KV_BF16
    dims = CDims(seq_lens.shape[0], q_tokens, Hkv, Hkv, D, P, num_pages, block_table.shape[1], 0, kv,
                 KBAR_F32)
    fp8 = kv == KV_FP8_E4M3
    _check(load().spattn_hca_pool(ctypes.byref(dims), _p(k_cache), _p(v_cache),
                                  _p(k_scale) if fp8 else None, _p(v_scale) if fp8 else None,
                                  _p(block_table), _p(old_lens), _p(seq_lens), _p(khat), _p(vhat),
                                  _stream(stream)))


def hca_workspace(q, k_cache, block_table) -> torch.Tensor:
    """Workspace of hca_attend for these shapes (spattn_hca_workspace_size)."""
    dims = dims_for(q, k_cache, block_table)
    n = load().spattn_hca_workspace_size(ctypes.byref(dims))
    if n == 0:
        raise SpattnError(1, "invalid dims")
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def hca_attend(q, khat, vhat, seq_lens, out, lse, params: Params, *, k_cache, block_table, workspace=None,
               stream=None, merge_with=None):
    """Dense attention of every query row over its visible pooled entries.
    ``merge_with=(out_other, lse_other)``: the result merged with another
    branch's (spattn_hca_attend_merge; lse may be None).  ``workspace``:
    from hca_workspace(); allocated here when not given."""
    dims = dims_for(q, k_cache, block_table)
    ws = workspace if workspace is not None else hca_workspace(q, k_cache, block_table)
    tail = [_p(ws), ws.numel() * ws.element_size(), _stream(stream)]
    if merge_with is None:
        _check(load().spattn_hca_attend(ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(khat),
                                        _p(vhat), _p(seq_lens), _p(out), _p(lse), *tail))
    else:
        _check(load().spattn_hca_attend_merge(ctypes.byref(dims), ctypes.byref(params.c()), _p(q), _p(khat),
                                              _p(vhat), _p(seq_lens), _p(merge_with[0]), _p(merge_with[1]),
                                              _p(out), _p(lse), *tail))


def lse_merge(out_a, lse_a, out_b, lse_b, out, lse=None, stream=None):
    """One softmax over two disjoint key sets from two partial results
    ([B][Tq][Hq][128] outputs, [B][Tq][Hq] log-sum-exps)."""
    B, Tq, Hq, D = out_a.shape
    dims = CDims(B, Tq, Hq, 1, D, 64, 1, 1, 0, KV_BF16, KBAR_F32)
    _check(load().spattn_lse_merge(ctypes.byref(dims), _p(out_a), _p(lse_a), _p(out_b), _p(lse_b), _p(out),
                                   _p(lse), _stream(stream)))


def device_status(stream=None) -> int:
    """Synchronise, read and clear the device status word (SPATTN_DEV_* bits)."""
    v = ctypes.c_int32(0)
    _check(load().spattn_get_device_status(ctypes.byref(v), _stream(stream)))
    return v.value


def version() -> str:
    return load().spattn_version().decode()
