"""The C-ABI library on the host: it loads, exports every entry point the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from block_sparse_kv_spattn_b200 import build, spattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return spattn.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "spattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spattn_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(spattn.EXPORTS)


def test_only_the_abi_is_exported():
    out = os.popen(f"nm -D --defined-only {spattn.LIB_PATH}").read().split("\n")
    syms = [l.split()[-1] for l in out if l.strip() and l.split()[1] in ("T", "W")]
    assert syms and all(s.startswith("spattn_") for s in syms), syms


def _dims(**kw):
    d = dict(batch=2, q_tokens=1, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=64,
             num_pages=100, max_blocks_per_seq=50, max_sel=50, kv_dtype=0, kbar_dtype=0)
    d.update(kw)
    return spattn.CDims(*[d[n] for n, _ in spattn.CDims._fields_])


def test_required_max_sel_rule(lib):
    p = spattn.Params(mode="topp", top_p=0.9, max_ratio=0.15)
    d = _dims(max_blocks_per_seq=2048)
    # n_mid = 2045, k_max = floor(0.15 * 2045) = 306
    assert spattn.required_max_sel(d, p) == 3 + 306
    p = spattn.Params(mode="topk", top_k=8)
    assert spattn.required_max_sel(_dims(max_blocks_per_seq=64), p) == 11
    assert spattn.required_max_sel(_dims(max_blocks_per_seq=2, q_tokens=1), p) == 2
    p = spattn.Params(mode="topk", max_ratio=0.12)
    d = _dims(q_tokens=16, num_q_heads=32, max_blocks_per_seq=8192)
    assert spattn.required_max_sel(d, p) == 3 + min(8189, 16 * 982)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), 2), (dict(block_size=32), 2), (dict(num_q_heads=30), 1),
    (dict(num_kv_heads=3, num_q_heads=3), 2), (dict(batch=0), 1), (dict(kv_dtype=7), 1),
    (dict(q_tokens=1025, num_q_heads=32), 2),          # 4100 query rows per KV head
])
def test_bad_dims_rejected(lib, kw, status):
    d = _dims(**kw)
    p = spattn.Params()
    assert lib.spattn_required_max_sel(ctypes.byref(d), ctypes.byref(p.c())) == -1
    assert lib.spattn_decode_workspace_size(ctypes.byref(d), ctypes.byref(p.c())) == 0
    st = lib.spattn_block_scores(ctypes.byref(d), ctypes.byref(p.c()), None, None, None, None, None, None)
    assert st == status
    assert lib.spattn_last_error()


@pytest.mark.parametrize("kw", [dict(mode="topp", top_p=0.0), dict(mode="topp", top_p=1.5),
                                dict(max_ratio=1.5), dict(sink_blocks=-1), dict(top_k=-2),
                                dict(sm_scale=float("inf"))])
def test_bad_params_rejected(lib, kw):
    d = _dims()
    p = spattn.Params(**kw)
    assert lib.spattn_select(ctypes.byref(d), ctypes.byref(p.c()), None, None, None, None, None) == 1


def test_null_pointers_rejected(lib):
    d, p = _dims(), spattn.Params(top_k=4)
    dummy = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    assert lib.spattn_compress_keys(ctypes.byref(d), None, None, dummy, None, dummy, dummy, None) == 1
    assert lib.spattn_select(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, None, dummy, None) == 1
    d.kv_dtype = 1
    assert lib.spattn_decode_selected(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, None,
                                      None, dummy, dummy, dummy, dummy, dummy, dummy, 1 << 30, None) == 1
    assert b"k_scale" in lib.spattn_last_error()


def test_small_max_sel_and_workspace_rejected(lib):
    d, p = _dims(max_sel=5), spattn.Params(top_k=8)
    dummy = ctypes.c_void_p(256)
    assert lib.spattn_select(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, dummy, None) == 1
    assert b"max_sel" in lib.spattn_last_error()
    d.max_sel = 50
    st = lib.spattn_decode_selected(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, None,
                                    None, dummy, dummy, dummy, dummy, dummy, dummy, 16, None)
    assert st == 4


def test_version(lib):
    assert "sm_100a" in spattn.version()


def test_hca_entry_points_validate_on_the_host(lib):
    """The HCA entries and the lse variant check sizes, pointers and
    alignment before enqueueing anything."""
    d, p = _dims(max_blocks_per_seq=51), spattn.Params(top_k=4)
    dummy, odd = ctypes.c_void_p(256), ctypes.c_void_p(260)
    assert lib.spattn_hca_entries(ctypes.byref(d)) == 26          # ceil(51 / 2)
    assert lib.spattn_hca_entries(ctypes.byref(_dims(head_dim=64))) == -1
    assert lib.spattn_hca_pool(ctypes.byref(d), dummy, dummy, None, None, dummy, None, dummy, None, dummy,
                               None) == 1
    d.kv_dtype = 1
    assert lib.spattn_hca_pool(ctypes.byref(d), dummy, dummy, None, None, dummy, None, dummy, dummy, dummy,
                               None) == 1
    assert b"scale" in lib.spattn_last_error()
    d.kv_dtype = 0
    assert lib.spattn_hca_pool(ctypes.byref(d), dummy, dummy, None, None, dummy, None, dummy, odd, dummy,
                               None) == 1
    assert b"aligned" in lib.spattn_last_error()
    assert lib.spattn_hca_attend(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, dummy, dummy,
                                 None, dummy, 1 << 30, None) == 1
    need = lib.spattn_hca_workspace_size(ctypes.byref(d))
    assert need >= 2 * 8 * 16 * 4 * 128 * 4     # B * Hkv * max split * rows * d floats
    assert lib.spattn_hca_attend(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, dummy, dummy,
                                 dummy, dummy, need - 1, None) == 4
    assert lib.spattn_hca_attend_merge(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, dummy, None,
                                       dummy, dummy, None, dummy, need, None) == 1
    assert lib.spattn_lse_merge(ctypes.byref(d), dummy, dummy, dummy, None, dummy, None, None) == 1
    assert lib.spattn_lse_merge(ctypes.byref(_dims(head_dim=96)), dummy, dummy, dummy, dummy, dummy, None,
                                None) == 2
    st = lib.spattn_decode_selected_lse(ctypes.byref(d), ctypes.byref(p.c()), dummy, dummy, dummy, None,
                                        None, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 16, None)
    assert st == 4


@pytest.mark.parametrize("kw,records", [
    (dict(), 4),                                                  # bf16, 4 rows: one record per softmax warp
    (dict(q_tokens=4, num_q_heads=16, num_kv_heads=2), 1),        # 32 rows: the many-row kernel, one record
    (dict(kv_dtype=1), 2),                                        # fp8: the many-row kernel, two softmax halves
])
def test_workspace_size_is_the_documented_layout(lib, kw, records):
    """The scores (B x Tq x Hkv x max_blocks fp32) when spattn_decode keeps
    them in the workspace, then split-KV partials (C_max + B * Hkv) x R
    records of rows x (d + 2) fp32, C_max = 320; each part 256-byte
    aligned."""
    d = _dims(**kw)
    p = spattn.Params(top_k=4)

    def up(x):
        return (x + 255) // 256 * 256

    rows = d.q_tokens * d.num_q_heads // d.num_kv_heads
    slots = (320 + d.batch * d.num_kv_heads) * records
    scores = up(d.batch * d.q_tokens * d.num_kv_heads * d.max_blocks_per_seq * 4)
    want = scores + up(slots * rows * 128 * 4) + up(slots * rows * 2 * 4)
    assert lib.spattn_decode_workspace_size(ctypes.byref(d), ctypes.byref(p.c())) == want
