"""Failure detection on the GPU without a fault: the bounded wait every
pipeline stage of the kernels uses is made to run out (a barrier nothing
arrives on, tests/native/wait_timeout.cu, compiled from the kernels' own
header); it must give up after its limit, report SPATTN_DEV_WAIT_TIMEOUT in
the device status word, end the kernel normally, and leave the context
usable.  Bad data found on the device is reported the same way: a selected
block past the request's end is skipped and flagged, never trapped.
(Named so that pytest collects it after the parity tests.)"""
import os
import subprocess

import pytest
import torch

from block_sparse_kv_spattn_b200 import build as B
from block_sparse_kv_spattn_b200 import spattn
from block_sparse_kv_spattn_b200.workloads import WORKLOADS, make_inputs
from tests.parity import lib_params

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_bounded_wait_gives_up_and_reports(cuda, tmp_path):
    exe = str(tmp_path / "wait_timeout")
    subprocess.run([B._nvcc(), *B.ARCH, "-O2", "-std=c++17", "-I", B.CSRC, "-I", B.INCLUDE,
                    os.path.join(HERE, "native", "wait_timeout.cu"), "-o", exe], check=True, timeout=300)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")


def test_selected_block_past_the_end_is_flagged_not_trapped(cuda):
    w = WORKLOADS["tiny_4k_gqa4"]
    inp = make_inputs(w, device="cuda")
    params = lib_params(w)
    q, kc, vc, bt, sl = inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["seq_lens"]
    dims = spattn.dims_for(q, kc, bt)
    max_sel = spattn.required_max_sel(dims, params)
    nb = (int(sl[0]) + w.block_size - 1) // w.block_size
    sel_idx = torch.zeros((w.batch, w.num_kv_heads, max_sel), dtype=torch.int32, device="cuda")
    sel_count = torch.full((w.batch, w.num_kv_heads), 2, dtype=torch.int32, device="cuda")
    sel_idx[:, :, 0] = 0
    sel_idx[:, :, 1] = nb + 3          # past the request's end
    dims.max_sel = max_sel
    ws = spattn.alloc_workspace(dims, params, "cuda")
    out = torch.empty(tuple(q.shape), device="cuda")
    spattn.device_status()
    spattn.decode_selected(q, kc, vc, inp["k_scale"], inp["v_scale"], bt, sl, sel_idx, sel_count, out, ws, params)
    status = spattn.device_status()
    assert status & spattn.DEV_BAD_BLOCK
    assert torch.isfinite(out).all()
    # the context is intact: a correct call afterwards reports nothing
    sel_count.fill_(1)
    spattn.decode_selected(q, kc, vc, inp["k_scale"], inp["v_scale"], bt, sl, sel_idx, sel_count, out, ws, params)
    assert spattn.device_status() == 0
