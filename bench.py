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
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            try:
                rows.append((float(f[0]), float(f[1]), f[3:7]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


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
        if not anchored:
            torch.cuda.current_stream().wait_stream(side)
        if w.hca:
            torch.cuda.current_stream().wait_stream(side2)

    def attend():  # sparse attention + split merge
        if not w.hca:
            spattn.decode_selected(q, kc, vc, ks, vs, bt, sl, sel_idx, sel_count, out, ws, params)
        else:
            spattn.decode_selected(q, kc, vc, ks, vs, bt, sl, sel_idx, sel_count, out_s, ws, params, lse=lse_s)

    def hca():     # the HCA branch's attention and the merge of the two branches
        if w.hca:
            spattn.hca_attend(q, khat, vhat, sl, out, None, params, k_cache=kc, block_table=bt, workspace=hca_ws,
                              merge_with=(out_s, lse_s))

    # warm up eagerly once (sets kernel attributes), then capture graphs
    front()
    attend()
    hca()
    torch.cuda.synchronize()
    status = spattn.device_status()
    if status:
        raise RuntimeError(f"device status {status:#x}")
    # the whole step in one graph; events recorded as graph nodes time its
    # parts on the device (start, after the front, after the sparse
    # attention, after the HCA branch)
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step, stream=s):
            marks[0].record()
            front()
            marks[1].record()
            attend()
            marks[2].record()
            hca()
            marks[3].record()
    torch.cuda.current_stream().wait_stream(s)
    launches_per_step = 5          # compress, scores, select, attention, merge
    if w.hca:
        launches_per_step += 3     # hca_pool, hca_partial, hca_combine (merging the sparse result)

    for _ in range(args.warmup):
        flush_l2()
        g_step.replay()
    torch.cuda.synchronize()
    K = args.steps
    step_ms, attn_ms, hca_list = [], [], []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    smi_id = (f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
              if hasattr(props, "pci_bus_id") else str(local_rank))
    with Clocks(smi_id) as clk:
        t_wall = time.perf_counter()
        for i in range(K):
            flush_l2()
            g_step.replay()
            marks[3].synchronize()
            step_ms.append(marks[0].elapsed_time(marks[3]))
            attn_ms.append(marks[1].elapsed_time(marks[2]))
            hca_list.append(marks[2].elapsed_time(marks[3]))
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    hca_ms = sum(hca_list) / K
    front_ms = sum(st - at - hc for st, at, hc in zip(step_ms, attn_ms, hca_list)) / K
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
    queries = B * Tq * world / (ms_per_step * 1e-3)
    e2e_value = all_bytes / (e2e_total_ms / K * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8" if w.kv_fp8 else "bf16",
        "data": "synthetic (seeded; power-law block importance)",
        "config": {"workload": w.name, "batch": B, "q_tokens": Tq, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": Hkv, "seq_len": w.seq_len, "block": w.block_size,
                   "sink_blocks": w.sink_blocks, "local_blocks": w.local_blocks,
                   "selection": (f"{w.mode} p={w.top_p} cap={w.max_ratio}" if w.mode == "topp" else
                                 f"{w.mode} p={w.top_p} cap={w.min_ratio}-{w.max_ratio} by anchors"
                                 if w.mode == "topp_anchor" else f"{w.mode} k={w.top_k} ratio={w.max_ratio}"),
                   "l2": "flushed between steps (512 MB write, then a 512 MB read so the flush's dirty lines are written back; outside the timed events)",
                   "parallelism": f"independent replicas x{world}"},
        "hbm_fraction": round(value / peak, 4),
        "queries_per_s": round(queries, 1),
        "bytes_per_step": bts,
        "roofline": {"kernel": attn_label(w),
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": None if traffic is None else int(traffic),
                     "ms_per_launch": round(attn_ms_mean, 5)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": q.numel() * 2 + sl.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 4},
        "front_ms": round(front_ms, 5),
        "gpu_launches": K * launches_per_step,
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


def cpu_baseline(inp, bts, gpu_ms):
    """The float64 oracle on this host's cores, on a bounded sample: all KV
    heads of request 0 (scores, selection, attention; compressed keys are
    computed outside the timing), scaled to the whole step."""
    import oracle
    from tests.oracle_io import bits16, cache_bytes, dims_of, params_of
    from tests.parity import subproblem

    w = inp["workload"]
    sub = subproblem(inp, 0)
    dims = dims_of(sub)
    par = params_of(w)
    qh, kh, vh = bits16(sub["q"]), cache_bytes(sub["k_cache"]), cache_bytes(sub["v_cache"])
    ksc, vsc = sub["k_scale"].cpu().numpy(), sub["v_scale"].cpu().numpy()
    bt, sl = sub["block_table"].cpu().numpy(), sub["seq_lens"].cpu().numpy()
    kbar = oracle.compress_keys(dims, kh, ksc, bt, sl)
    if w.hca:   # pooled entries, like the compressed keys, outside the timing
        khat, vhat = oracle.hca_pool(dims, kh, vh, ksc, vsc, bt, sl)
    times = []
    t_end = time.perf_counter() + 10.0
    while time.perf_counter() < t_end or not times:
        t0 = time.perf_counter()
        sc = oracle.block_scores(dims, par, qh, kbar, bt, sl)
        sel, cnt, _ = oracle.select(dims, par, sc, sl)
        o_s = oracle.attend(dims, par, qh, kh, vh, ksc, vsc, bt, sl, sel, cnt, with_lse=w.hca)
        if w.hca:
            oracle.lse_merge(*o_s, *oracle.hca_attend(dims, par, qh, khat, vhat, sl))
        times.append(time.perf_counter() - t0)
    per_req = statistics.median(times)
    step_s = per_req * w.batch
    return {"value": round(bts["total"] / step_s / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"request 0 of {w.batch} (all {w.num_kv_heads} KV heads{', both branches' if w.hca else ''}), "
                      f"{len(times)} runs, "
                      f"median {per_req:.3f} s, scaled x{w.batch} to the step",
            "ms_per_step": round(step_s * 1e3, 3), "gpu_speedup": round(step_s * 1e3 / gpu_ms, 1)}


def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only, bounded per-step sample."""
    if rank != 0:
        return None
    import oracle
    from tests.oracle_io import bits16, cache_bytes, dims_of, params_of
    from tests.parity import subproblem

    w = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, device=dev)
    par = params_of(w)
    subs = []
    # per step: one (request, KV head) unit of the workload, cycling
    for b in range(min(w.batch, 2)):
        sub = subproblem(inp, b)
        dims = dims_of(sub)
        qh, kh, vh = bits16(sub["q"]), cache_bytes(sub["k_cache"]), cache_bytes(sub["v_cache"])
        ksc, vsc = sub["k_scale"].cpu().numpy(), sub["v_scale"].cpu().numpy()
        bt, sl = sub["block_table"].cpu().numpy(), sub["seq_lens"].cpu().numpy()
        kbar = oracle.compress_keys(dims, kh, ksc, bt, sl)
        hat = oracle.hca_pool(dims, kh, vh, ksc, vsc, bt, sl) if w.hca else None
        subs.append((dims, qh, kh, vh, ksc, vsc, bt, sl, kbar, hat))
    # with the HCA branch a unit is a whole request (its dense attention
    # covers all KV heads at once); otherwise one (request, KV head)
    units = w.batch * (1 if w.hca else w.num_kv_heads)

    def one(i):
        dims, qh, kh, vh, ksc, vsc, bt, sl, kbar, hat = subs[i % len(subs)]
        sc = oracle.block_scores(dims, par, qh, kbar, bt, sl)
        sel, cnt, _ = oracle.select(dims, par, sc, sl)
        if w.hca:
            o_s = oracle.attend(dims, par, qh, kh, vh, ksc, vsc, bt, sl, sel, cnt, with_lse=True)
            oracle.lse_merge(*o_s, *oracle.hca_attend(dims, par, qh, hat[0], hat[1], sl))
            return int(cnt[0].sum())
        h = (i // len(subs)) % w.num_kv_heads
        oracle.attend(dims, par, qh, kh, vh, ksc, vsc, bt, sl, sel, cnt, units=[(0, h)])
        return int(cnt[0, h])

    for i in range(args.warmup):
        one(i)
    times, kept = [], 0
    budget = time.perf_counter() + 150.0
    for i in range(args.steps):
        t0 = time.perf_counter()
        kept += one(i)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > budget:
            break
    per_unit = statistics.mean(times)
    step_s = per_unit * units
    # bytes of a full step at the sampled units' mean kept count
    P, D = w.block_size, w.head_dim
    elt = 1 if w.kv_fp8 else 2
    mean_kept = kept / len(times)
    nbs = [(int(L) + P - 1) // P for L in inp["seq_lens"].tolist()]
    n_mid = sum(max(0, nb - w.sink_blocks - w.local_blocks) for nb in nbs)
    total = units * mean_kept * P * D * elt * 2 + n_mid * w.num_kv_heads * D * 4 + inp["q"].numel() * 6
    if w.hca:
        total += step_bytes(inp, torch.zeros(1))["hca"]
    value = total / step_s / 1e9
    what = "request" if w.hca else "(request, KV head)"
    sample = (f"{len(times)} steps x one {what} unit of {units} (scores, selection, attention"
              f"{', HCA branch and merge' if w.hca else ''} in float64), scaled x{units} to the step")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": len(times), "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; power-law block importance)",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


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
