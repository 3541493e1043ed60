"""Benchmark: block-sparse decode attention at 128K context on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME]

One step is one pass of the whole decode path over the workload's batch:
incremental key compression of each request's tail block (on a forked
graph branch: the tail block is local, never scored), block scores,
selection (sink + local + top-p/top-k), sparse attention and the split
merge (and, for the HCA workloads, the dense branch over pooled 128-token
entries merged with the sparse one), all through the C ABI, captured once
into one CUDA graph per step and replayed.  Event-record nodes inside the
graph time the step and its parts on the device.  Inputs are seeded
synthetic data resident in HBM; L2 is flushed (a 512 MB write, then a 512 MB
read that writes the flush's dirty lines back) before every timed step,
outside the timed events.

Metric: selected-KV HBM GB/s = algorithmic bytes of a step (kept K+V tiles,
fp8 scales, compressed keys of the scored middle blocks, q, out) / step time,
aggregated over ranks; decode queries/s alongside.  Under torchrun each rank
runs its own independent batch (weak scaling, no collective on the data
path); the step time is the max over ranks.

--impl reference times the float64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_kv_spattn_b200.workloads import BENCH_WORKLOAD, WORKLOADS, make_inputs  # noqa: E402

METRIC = "selected-KV HBM GB/s (% of ~8 TB/s) and decode queries/s at 128K ctx, 1 B200"
FLUSH_BYTES = 512 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")
# the sources of the kernel the traffic capture covers (attn_tc_kernel)
ATTN_SOURCES = ["common.cuh", "attention.cuh", "tcgen05.cuh", "attention_tc.cuh"]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _tensor_peak():
    """Dense bf16 TFLOP/s sustained under the power cap (the attention is
    timed inside a long run of steps)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except Exception:
        return 1400.0, "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_kv_spattn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def attn_label(w) -> str:
    """The attention kernels one decode_selected call launches (timed together)."""
    rows = w.q_tokens * (w.num_q_heads // w.num_kv_heads)
    if not w.kv_fp8 and rows <= 16:
        rq = 4 if rows <= 4 else (8 if rows <= 8 else 16)
        return f"attention (attn_tc_kernel<{rq}> on tcgen05 + merge_kernel, one decode_selected call)"
    return (f"attention (attn_tcw_kernel<{'fp8' if w.kv_fp8 else 'bf16'}> on tcgen05, query rows on M, "
            f"+ merge_kernel, one decode_selected call)")


def measured_traffic(w, units_in_launch: float):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    capture, scaled to this launch; None if this workload runs another
    kernel or the kernel's sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except Exception:
        return None
    if t.get("kernel", "") not in attn_label(w) or t.get("source_sha") != attn_source_hash():
        return None
    return t["dram_bytes_per_launch"] * units_in_launch / t["units_per_launch"]


class Clocks:
    """SM clock and clock-event reasons sampled during a region, read-only:
    an NVML reader thread (a sample every ~0.5 ms, so that even a timed loop
    of a few milliseconds has samples), else nvidia-smi every 50 ms."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, pci_bus_id: str):
        self.bus = pci_bus_id
        self.rows = []
        self.source = None

    def __enter__(self):
        import threading
        self.rows, self.stop = [], threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def sample():
                while not self.stop.is_set():
                    try:
                        self.rows.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                          int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        break
                    time.sleep(0.0005)

            self.source = "nvml"
        except Exception:
            self.source = "nvidia-smi"

            def sample():
                q = "clocks.sm,clocks.max.sm,clocks_event_reasons.active"
                try:
                    proc = subprocess.Popen(["nvidia-smi", "--id=" + self.bus, f"--query-gpu={q}",
                                             "--format=csv,noheader,nounits", "-lms", "50"],
                                            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                except Exception:
                    return
                for line in proc.stdout:
                    f = [x.strip() for x in line.split(",")]
                    try:
                        self.max_mhz = float(f[1])
                        self.rows.append((float(f[0]), int(f[2], 16)))
                    except (ValueError, IndexError):
                        pass
                    if self.stop.is_set():
                        break
                proc.terminate()

        self.thread = threading.Thread(target=sample, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        self.stop.set()
        self.thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return None
        mask = 0
        for _, r in self.rows:
            mask |= r
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": getattr(self, "max_mhz", None),
                "reasons": [n for n, bit in self.REASONS if mask & bit], "samples": len(self.rows),
                "source": self.source, "window": "the timed loop"}


def step_bytes(inp, sel_count: torch.Tensor) -> dict:
    """Algorithmic bytes of one step (one rank)."""
    w = inp["workload"]
    P, D, H = w.block_size, w.head_dim, w.num_kv_heads
    elt = 1 if w.kv_fp8 else 2
    kept = int(sel_count.sum())
    kv = kept * P * D * elt * 2 + (kept * 8 if w.kv_fp8 else 0)
    n_mid = sum(max(0, (int(L) + P - 1) // P - w.sink_blocks - w.local_blocks)
                for L in inp["seq_lens"].tolist())
    if w.mode == "topp_anchor":     # the anchor blocks are scored too
        n_mid += sum(min((int(L) + P - 1) // P, w.sink_blocks + w.local_blocks) for L in inp["seq_lens"].tolist())
    kbar = n_mid * H * D * (2 if w.kbar_bf16 else 4)
    q = inp["q"].numel() * 2
    out = inp["q"].numel() * 4
    d = dict(kv=kv, kbar=kbar, q=q, out=out, total=kv + kbar + q + out, kept_block_heads=kept)
    if w.hca:
        # HCA branch: the visible entries' K and V means (fp32, once per KV
        # head), the appended tokens' entries re-pooled (their K and V read,
        # two means written), and the sparse branch's result read back into
        # the merged output (its out read, the merged out written, its lse
        # written and read)
        T, lens = 2 * P, inp["seq_lens"].tolist()
        entries = sum((int(L) + T - 1) // T for L in lens)
        pooled = sum(int(L) - (max(int(L) - w.q_tokens, 0) // T) * T for L in lens) * H * D * elt * 2
        rows = inp["q"].numel() // D
        attend = entries * H * D * 4 * 2 + 2 * out + 2 * rows * 4
        hca = attend + pooled + len(lens) * H * D * 4 * 2
        d.update(hca=hca, hca_attend=attend, total=d["total"] + hca)
    return d


def attention_flops(inp, sel_idx: torch.Tensor, sel_count: torch.Tensor) -> int:
    """Algorithmic FLOPs of one sparse-attention launch: 4 d per (query row,
    visible kept token) pair (q.k and p.v, 2 d each).  Query token t of a
    chunk of Tq sits at position L - Tq + t and sees the kept positions up to
    its own; every query head of the group sees the same ones."""
    w = inp["workload"]
    P, D, Tq = w.block_size, w.head_dim, w.q_tokens
    G = w.num_q_heads // w.num_kv_heads
    cnt, idx = sel_count.cpu(), sel_idx.cpu().to(torch.int64)
    pairs = 0
    for b, L in enumerate(inp["seq_lens"].tolist()):
        lims = L - Tq + 1 + torch.arange(Tq, dtype=torch.int64)          # positions < lim are visible
        for h in range(w.num_kv_heads):
            start = idx[b, h, :int(cnt[b, h])] * P
            pairs += int((lims[:, None] - start[None, :]).clamp(0, P).sum()) * G
    return pairs * 4 * D


def graph_kernels(g) -> list:
    """Names of the kernel nodes of a captured step graph: every kernel one
    replay launches (event-record nodes are not kernels).  Read through the
    driver API, which sees the same graph object torch captured."""
    from cuda.bindings import driver as cu

    graph = cu.CUgraph(g.raw_cuda_graph())
    err, _, n = cu.cuGraphGetNodes(graph, 0)
    if err != cu.CUresult.CUDA_SUCCESS:
        raise RuntimeError(f"cuGraphGetNodes: {err}")
    err, nodes, n = cu.cuGraphGetNodes(graph, n)
    if err != cu.CUresult.CUDA_SUCCESS:
        raise RuntimeError(f"cuGraphGetNodes: {err}")
    names = []
    for nd in nodes[:n]:
        err, kind = cu.cuGraphNodeGetType(nd)
        if err != cu.CUresult.CUDA_SUCCESS or kind != cu.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
            continue
        name = "?"
        try:
            err, prm = cu.cuGraphKernelNodeGetParams(nd)
            if err == cu.CUresult.CUDA_SUCCESS:
                err, nm = cu.cuFuncGetName(prm.func)
                if err != cu.CUresult.CUDA_SUCCESS:   # a library kernel handle instead
                    err, nm = cu.cuKernelGetName(prm.kern)
                if err == cu.CUresult.CUDA_SUCCESS:
                    name = nm.decode() if isinstance(nm, bytes) else str(nm)
        except Exception:
            pass
        names.append(name)
    return names


def reduce_over_ranks(t: torch.Tensor, world: int) -> list:
    """[times..., bytes, bytes]: the first three (timed totals) take the max
    over ranks, the last two (bytes moved) the sum.  Every rank calls it."""
    if world > 1:
        mx = t[:3].clone()
        torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
        sm = t[3:].clone()
        torch.distributed.all_reduce(sm, op=torch.distributed.ReduceOp.SUM)
        t = torch.cat([mx, sm])
    return t.tolist()


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent batch."""
    return base + 1000 * rank


def run_native(args, rank, world, local_rank):
    from block_sparse_kv_spattn_b200 import spattn

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, device=dev, seed=rank_seed(w.seed, rank))
    q, kc, vc, ks, vs = inp["q"], inp["k_cache"], inp["v_cache"], inp["k_scale"], inp["v_scale"]
    bt, sl = inp["block_table"], inp["seq_lens"]
    params = spattn.Params(sink_blocks=w.sink_blocks, local_blocks=w.local_blocks, mode=w.mode,
                           top_k=w.top_k, top_p=w.top_p, max_ratio=w.max_ratio, min_ratio=w.min_ratio)
    dims = spattn.dims_for(q, kc, bt)
    max_sel = spattn.required_max_sel(dims, params)
    dims.max_sel = max_sel
    B, Tq, Hkv = w.batch, w.q_tokens, w.num_kv_heads
    kbar = torch.empty((kc.shape[0], Hkv, w.head_dim), dtype=torch.bfloat16 if w.kbar_bf16 else torch.float32,
                       device=dev)
    spattn.compress_keys(kc, ks, bt, sl, kbar, num_q_heads=w.num_q_heads, q_tokens=Tq)
    old_lens = (sl - Tq).clamp_min(0).to(torch.int32)
    scores = torch.empty((B, Tq, Hkv, bt.shape[1]), dtype=torch.float32, device=dev)
    sel_idx = torch.empty((B, Hkv, max_sel), dtype=torch.int32, device=dev)
    sel_count = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
    out = torch.empty(tuple(q.shape), dtype=torch.float32, device=dev)
    ws = spattn.alloc_workspace(dims, params, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    drain = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # evict: write 512 MB (> 126 MB L2), then read another 512 MB so the
        # flush's own dirty lines are written back before the timed work
        flush.zero_()
        drain.sum()

    # The step's appended tokens only touch the last local block(s): their
    # compressed keys are never scored (local blocks are always kept), so the
    # append-side compression runs on a forked branch beside scoring.
    assert Tq <= (w.local_blocks - 1) * w.block_size + 1, "append would touch a middle block"
    side, side2 = torch.cuda.Stream(), torch.cuda.Stream()

    anchored = w.mode == "topp_anchor"   # the local blocks are scored: compress first

    if w.hca:
        # HCA branch: pooled entries (all of them now; the step re-pools the
        # appended tokens' entries), its output / lse and the sparse lse
        G = spattn.hca_entries(bt)
        khat = torch.empty((B, Hkv, G, w.head_dim), dtype=torch.float32, device=dev)
        vhat = torch.empty_like(khat)
        spattn.hca_pool(kc, vc, ks, vs, bt, sl, khat, vhat)
        lse_s = torch.empty(tuple(q.shape[:3]), dtype=torch.float32, device=dev)
        out_s = torch.empty_like(out)
        hca_ws = spattn.hca_workspace(q, kc, bt)

    def front():   # scores + selection, with the tail block's compression beside them
        if anchored:
            spattn.compress_keys(kc, ks, bt, sl, kbar, old_lens=old_lens, num_q_heads=w.num_q_heads,
                                 q_tokens=Tq)
        else:
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                spattn.compress_keys(kc, ks, bt, sl, kbar, old_lens=old_lens, num_q_heads=w.num_q_heads,
                                     q_tokens=Tq)
        if w.hca:   # the appended tokens' pooled entries, on a branch of their own
            side2.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side2):
                spattn.hca_pool(kc, vc, ks, vs, bt, sl, khat, vhat, old_lens=old_lens, q_tokens=Tq)
        spattn.block_scores(q, kbar, bt, sl, scores, params, k_cache=kc)
        spattn.select(scores, sl, sel_idx, sel_count, params, q=q, k_cache=kc, block_table=bt)

    def join_branches():   # the branches forked in front() (and the marks), before the step's end
        if not anchored:
            torch.cuda.current_stream().wait_stream(side)
        torch.cuda.current_stream().wait_stream(marks_stream)

    def attend():  # sparse attention + split merge
        if not w.hca:
            spattn.decode_selected(q, kc, vc, ks, vs, bt, sl, sel_idx, sel_count, out, ws, params)
        else:
            spattn.decode_selected(q, kc, vc, ks, vs, bt, sl, sel_idx, sel_count, out_s, ws, params, lse=lse_s)

    def hca():     # the HCA branch's attention and the merge of the two branches
        if w.hca:
            torch.cuda.current_stream().wait_stream(side2)
            spattn.hca_attend(q, khat, vhat, sl, out, None, params, k_cache=kc, block_table=bt, workspace=hca_ws,
                              merge_with=(out_s, lse_s))

    # the marks between the step's parts are recorded on a branch of their
    # own, so that no kernel of the step waits behind an event node
    marks_stream = torch.cuda.Stream()

    def mark(ev):
        marks_stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(marks_stream):
            ev.record()

    # warm up eagerly once (sets kernel attributes), then capture graphs
    front()
    attend()
    hca()
    join_branches()
    torch.cuda.synchronize()
    status = spattn.device_status()
    if status:
        raise RuntimeError(f"device status {status:#x}")
    # the whole step in one graph; events recorded as graph nodes time its
    # parts on the device (start, after the front, after the sparse
    # attention, after the HCA branch and the joins).  The middle two are
    # leaves on a branch of their own (see mark()).
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g_step = torch.cuda.CUDAGraph(keep_graph=True)   # kept to list its kernel nodes
        with torch.cuda.graph(g_step, stream=s):
            marks[0].record()
            front()
            mark(marks[1])
            attend()
            mark(marks[2])
            hca()
            join_branches()
            marks[3].record()
    torch.cuda.current_stream().wait_stream(s)
    kernels_error = None
    try:
        step_kernels = graph_kernels(g_step)
        launches_per_step = len(step_kernels)
    except Exception as e:   # no driver bindings: the kernels a step is built from
        step_kernels, kernels_error = None, f"{type(e).__name__}: {e}"
        launches_per_step = 5 + (3 if w.hca else 0)
    g_step.instantiate()

    K = args.steps
    step_ms, attn_ms, hca_list, front_list = [], [], [], []
    props = torch.cuda.get_device_properties(dev)
    smi_id = (f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
              if hasattr(props, "pci_bus_id") else str(local_rank))
    for _ in range(args.warmup):
        flush_l2()
        g_step.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(smi_id) as clk:
        t_wall = time.perf_counter()
        for i in range(K):
            flush_l2()
            g_step.replay()
            marks[3].synchronize()
            step_ms.append(marks[0].elapsed_time(marks[3]))
            attn_ms.append(marks[1].elapsed_time(marks[2]))
            hca_list.append(marks[2].elapsed_time(marks[3]))
            front_list.append(marks[0].elapsed_time(marks[1]))
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
        if world > 1:
            torch.distributed.barrier()
    hca_ms = sum(hca_list) / K
    front_ms = sum(front_list) / K
    total_ms = sum(step_ms)
    bts = step_bytes(inp, sel_count)
    status = spattn.device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after the timed region")

    # e2e: q / seq_lens in from pinned host memory, out back, every step
    q_h = q.cpu().pin_memory()
    sl_h = sl.cpu().pin_memory()
    out_h = torch.empty(tuple(out.shape), dtype=out.dtype).pin_memory()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        flush_l2()
        e2e_ev[i][0].record()
        q.copy_(q_h, non_blocking=True)
        sl.copy_(sl_h, non_blocking=True)
        g_step.replay()
        out_h.copy_(out, non_blocking=True)
        e2e_ev[i][1].record()
    torch.cuda.synchronize()
    e2e_ms = sum(e[0].elapsed_time(e[1]) for e in e2e_ev)

    t = torch.tensor([total_ms, sum(attn_ms), e2e_ms, float(bts["total"]), float(bts["kv"] + bts["q"] + bts["out"])],
                     dtype=torch.float64, device=dev)
    total_ms, attn_total_ms, e2e_total_ms, all_bytes, _ = reduce_over_ranks(t, world)
    if rank != 0:
        return None
    ms_per_step = total_ms / K
    value = all_bytes / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    attn_ms_mean = attn_total_ms / K
    attn_bytes = bts["kv"] + bts["q"] + bts["out"]     # one rank's launch
    achieved = attn_bytes / (attn_ms_mean * 1e-3) / 1e9
    traffic = measured_traffic(w, bts["kept_block_heads"])
    # the attention's bound: its HBM bytes at the copy peak, or its FLOPs at
    # the tensor peak, whichever takes longer
    flops = attention_flops(inp, sel_idx, sel_count)
    tpeak, tpeak_kind = _tensor_peak()
    tensor_bound = flops / (tpeak * 1e12) > attn_bytes / (peak * 1e9)
    tflops = flops / (attn_ms_mean * 1e-3) / 1e12
    queries = B * Tq * world / (ms_per_step * 1e-3)
    e2e_value = all_bytes / (e2e_total_ms / K * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8" if w.kv_fp8 else "bf16",
        "data": "synthetic (seeded; power-law block importance)",
        "config": workload_config(w, world),
        "hbm_fraction": round(value / peak, 4),
        "queries_per_s": round(queries, 1),
        "bytes_per_step": bts,
        "roofline": ({"kernel": attn_label(w),
                      "bound": "tensor", "achieved": round(tflops, 1), "peak": tpeak, "peak_kind": tpeak_kind,
                      "unit": "TFLOP/s", "frac": round(tflops / tpeak, 4),
                      "traffic": None if traffic is None else int(traffic),
                      "ms_per_launch": round(attn_ms_mean, 5), "flops": flops,
                      "hbm": {"achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                              "frac": round(achieved / peak, 4)}}
                     if tensor_bound else
                     {"kernel": attn_label(w),
                      "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                      "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                      "unit": "GB/s", "frac": round(achieved / peak, 4),
                      "traffic": None if traffic is None else int(traffic),
                      "ms_per_launch": round(attn_ms_mean, 5), "flops": flops,
                      "tensor": {"achieved": round(tflops, 1), "peak": tpeak, "unit": "TFLOP/s",
                                 "frac": round(tflops / tpeak, 4)}}),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": q.numel() * 2 + sl.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 4},
        "front_ms": round(front_ms, 5),
        "gpu_launches": K * launches_per_step,
        "step_kernels": sorted(step_kernels) if step_kernels is not None else kernels_error,
        "clocks": clk.summary(),
        "wall_s": round(t_wall, 3),
    }
    if w.hca:
        line["hca"] = {"kernels": "hca_partial_kernel + hca_combine_kernel merging the sparse result "
                                  "(timed apart from the sparse branch)",
                       "ms_per_step": round(hca_ms, 5), "bytes": bts["hca_attend"],
                       "achieved": round(bts["hca_attend"] / (hca_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                       "frac": round(bts["hca_attend"] / (hca_ms * 1e-3) / 1e9 / peak, 4)}
    if w.kbar_bf16:
        line["recall_vs_fp32_kbar"] = kbar_recall(inp, params, sel_idx, sel_count, dev)
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(inp, bts, ms_per_step)
    return line


def kbar_recall(inp, params, sel_idx, sel_count, dev) -> float:
    """Low-precision scoring, measured (outside the timed region): the share
    of the middle blocks selected from fp32 compressed keys that the bf16
    keys' selection also keeps, over every (request, KV head)."""
    from block_sparse_kv_spattn_b200 import spattn
    w = inp["workload"]
    q, kc, bt, sl = inp["q"], inp["k_cache"], inp["block_table"], inp["seq_lens"]
    kb32 = torch.empty((kc.shape[0], w.num_kv_heads, w.head_dim), dtype=torch.float32, device=dev)
    spattn.compress_keys(kc, inp["k_scale"], bt, sl, kb32, num_q_heads=w.num_q_heads, q_tokens=w.q_tokens)
    sc = torch.empty((w.batch, w.q_tokens, w.num_kv_heads, bt.shape[1]), dtype=torch.float32, device=dev)
    si = torch.empty_like(sel_idx)
    cnt = torch.empty_like(sel_count)
    spattn.block_scores(q, kb32, bt, sl, sc, params, k_cache=kc)
    spattn.select(sc, sl, si, cnt, params, q=q, k_cache=kc, block_table=bt)
    torch.cuda.synchronize()
    P = w.block_size
    hit = total = 0
    for b in range(w.batch):
        nb = (int(sl[b]) + P - 1) // P
        anchors = set(range(w.sink_blocks)) | set(range(nb - w.local_blocks, nb))
        for h in range(w.num_kv_heads):
            ref = set(si[b, h, :int(cnt[b, h])].tolist()) - anchors
            got = set(sel_idx[b, h, :int(sel_count[b, h])].tolist()) - anchors
            hit += len(ref & got)
            total += len(ref)
    return round(hit / max(1, total), 5)


def oracle_request(inp, b, heads=None, last_tokens=None):
    """The float64 oracle's work for request b of the batch: scores,
    selection and attention for all its KV heads, or only for the KV heads
    listed in `heads` (scores and selection still cover every head: they are
    a small part of the work); for the HCA workloads also the dense branch
    and the merge.  `last_tokens`: the attention of a chunk's last n query
    tokens only (at their own positions, over the selection of the whole
    chunk).  Compressed keys and pooled entries are computed here, outside
    the timed call, as the GPU step only re-compresses the appended tail.
    Returns run() -> kept block-heads of the attended heads."""
    import dataclasses

    import numpy as np
    import oracle
    from oracle.marshal import bits16, cache_bytes, dims_of, params_of, subproblem

    w = inp["workload"]
    sub = subproblem(inp, b)
    dims = dims_of(sub)
    par = params_of(w)
    qh, kh, vh = bits16(sub["q"]), cache_bytes(sub["k_cache"]), cache_bytes(sub["v_cache"])
    ksc, vsc = sub["k_scale"].cpu().numpy(), sub["v_scale"].cpu().numpy()
    bt, sl = sub["block_table"].cpu().numpy(), sub["seq_lens"].cpu().numpy()
    kbar = oracle.compress_keys(dims, kh, ksc, bt, sl)
    hat = oracle.hca_pool(dims, kh, vh, ksc, vsc, bt, sl) if w.hca else None
    units = None if heads is None else [(0, h) for h in heads]
    dims_a, q_a = dims, qh
    if last_tokens is not None and last_tokens < w.q_tokens:
        # token t' of the last n sits at L - n + t' = L - Tq + (Tq - n + t')
        dims_a = dataclasses.replace(dims, q_tokens=last_tokens)
        q_a = np.ascontiguousarray(qh[:, w.q_tokens - last_tokens:])

    def run():
        sc = oracle.block_scores(dims, par, qh, kbar, bt, sl)
        sel, cnt, _ = oracle.select(dims, par, sc, sl)
        o_s = oracle.attend(dims_a, par, q_a, kh, vh, ksc, vsc, bt, sl, sel, cnt, with_lse=w.hca, units=units)
        if w.hca:
            oracle.lse_merge(*o_s, *oracle.hca_attend(dims, par, qh, hat[0], hat[1], sl))
        return int(cnt.sum()) if heads is None else int(sum(cnt[0, h] for h in heads))

    return run


def _time_runs(run, seconds, min_runs=1, max_runs=None):
    times = []
    t_end = time.perf_counter() + seconds
    while (time.perf_counter() < t_end or len(times) < min_runs) and (max_runs is None or len(times) < max_runs):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    return times


def oracle_sample(inp) -> dict:
    """The bounded sample of a step's oracle work that both host legs time:
    request 0 (scores, selection, attention); when one request would take
    more than ~10 s, its KV head 0 alone; when that would too (long
    chunks), the attention of the chunk's last few query tokens of KV head 0
    at their own positions over the whole chunk's selection.  Returns run()
    (-> kept block-heads of the attended heads), scale (sample -> step
    time), kept_scale (the attended heads' kept count -> the step's), the
    threads the sample keeps busy, and a description."""
    import oracle

    w = inp["workload"]
    H, Tq = w.num_kv_heads, w.q_tokens
    # one query token of KV head 0: the whole unit is at most Tq times that
    t_tok = min(_time_runs(oracle_request(inp, 0, heads=[0], last_tokens=1), 0.0, min_runs=1, max_runs=1))
    t_unit = t_tok * Tq
    whole = w.hca or H == 1 or t_unit * H <= 10.0   # (the HCA branch covers every head at once)
    n_tok = Tq if t_unit <= 10.0 else max(1, min(Tq, int(10.0 / t_tok)))
    what = (f"request 0 of {w.batch} (all {H} KV heads{', both branches' if w.hca else ''})" if whole
            else f"KV head 0 of request 0 (one of {w.batch * H} (request, KV head) units)" if n_tok == Tq
            else (f"the last {n_tok} of {Tq} query tokens of KV head 0 of request 0 (one of {w.batch * H} "
                  f"(request, KV head) units; selection over the whole chunk)"))
    return {"run": oracle_request(inp, 0) if whole else oracle_request(inp, 0, heads=[0], last_tokens=n_tok),
            "scale": w.batch if whole else w.batch * H * Tq / n_tok,
            "kept_scale": w.batch if whole else w.batch * H,
            # the oracle's attention runs its (request, KV head) units in parallel
            "cores": min(oracle.num_threads(), H if whole else 1),
            "what": what}


def cpu_baseline(inp, bts, gpu_ms):
    """The float64 oracle on this host's cores on the bounded sample of
    oracle_sample(), about 10 s of runs, median scaled to the whole step;
    then a few runs on one core, when they fit in ~30 s."""
    import oracle

    cores = oracle.num_threads()
    smp = oracle_sample(inp)
    run, scale, used = smp["run"], smp["scale"], smp["cores"]
    times = _time_runs(run, 10.0)
    per = statistics.median(times)
    step_s = per * scale
    line = {"value": round(bts["total"] / step_s / 1e9, 4), "unit": "GB/s", "cores": used,
            "host_threads": cores, "kind": "oracle",
            "sample": f"{smp['what']}, {len(times)} runs, median {per:.3f} s, scaled x{scale:g} to the step",
            "ms_per_step": round(step_s * 1e3, 3), "gpu_speedup": round(step_s * 1e3 / gpu_ms, 1)}
    # one core: the same sample, if about 5 runs fit in ~30 s
    if per * used * 5 <= 30.0 or used == 1:
        oracle.set_num_threads(1)
        try:
            t1 = _time_runs(run, 6.0, min_runs=1, max_runs=5)
        finally:
            oracle.set_num_threads(cores)
        step1_s = statistics.median(t1) * scale
        line["one_core"] = {"value": round(bts["total"] / step1_s / 1e9, 5), "unit": "GB/s", "cores": 1,
                            "ms_per_step": round(step1_s * 1e3, 3),
                            "sample": f"the same sample, {len(t1)} runs on one thread, scaled x{scale:g}"}
    return line


def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only.  One step = one run of
    the native arm's cpu_baseline sample (oracle_sample: request 0, or one of
    its KV heads, or the last tokens of one, on every core), scaled to the
    batch.  Bounded to about 150 s of timed work."""
    if rank != 0:
        return None
    import oracle

    w = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, device=dev)
    smp = oracle_sample(inp)
    run = smp["run"]
    for _ in range(args.warmup):
        run()
    times, kept = [], 0
    budget = time.perf_counter() + 150.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        kept += run()
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > budget:
            break
    per = statistics.median(times)
    step_s = per * smp["scale"]
    # bytes of a full step at the sample's kept count
    P, D = w.block_size, w.head_dim
    elt = 1 if w.kv_fp8 else 2
    kept_step = kept / len(times) * smp["kept_scale"]
    nbs = [(int(L) + P - 1) // P for L in inp["seq_lens"].tolist()]
    n_mid = sum(max(0, nb - w.sink_blocks - w.local_blocks) for nb in nbs)
    total = (kept_step * P * D * elt * 2 + (kept_step * 8 if w.kv_fp8 else 0)
             + n_mid * w.num_kv_heads * D * (2 if w.kbar_bf16 else 4) + inp["q"].numel() * 6)
    if w.hca:
        total += step_bytes(inp, torch.zeros(1))["hca"]
    value = total / step_s / 1e9
    sample = (f"{len(times)} steps x {smp['what']} (scores, selection, attention"
              f"{', HCA branch and merge' if w.hca else ''} in float64), median scaled x{smp['scale']:g}")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": len(times), "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; power-law block importance)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s",
                         "cores": smp["cores"], "host_threads": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def workload_config(w, world: int) -> dict:
    return {"workload": w.name, "batch": w.batch, "q_tokens": w.q_tokens, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "seq_len": w.seq_len, "block": w.block_size,
            "sink_blocks": w.sink_blocks, "local_blocks": w.local_blocks,
            "selection": (f"{w.mode} p={w.top_p} cap={w.max_ratio}" if w.mode == "topp" else
                          f"{w.mode} p={w.top_p} cap={w.min_ratio}-{w.max_ratio} by anchors"
                          if w.mode == "topp_anchor" else f"{w.mode} k={w.top_k} ratio={w.max_ratio}"),
            "l2": "flushed between steps (512 MB write, then a 512 MB read so the flush's dirty lines are "
                  "written back; outside the timed events)",
            "parallelism": f"independent replicas x{world}"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=sorted(WORKLOADS))
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "native":
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_native(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
