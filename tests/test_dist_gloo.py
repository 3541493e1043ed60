"""The multi-rank host logic of bench.py on CPU ranks (gloo, world size 2):
timed totals reduce by max over ranks, bytes by sum, and every rank draws
its own batch."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_kv_spattn_b200.workloads import WORKLOADS, make_inputs

        t = torch.tensor([10.0 + rank, 5.0 - rank, 7.0 * (rank + 1), 100.0 * (rank + 1), 3.0],
                         dtype=torch.float64)
        red = bench.reduce_over_ranks(t, world)
        w = WORKLOADS["tiny_4k_gqa4"].replace(seq_len=64 * 8)
        inp = make_inputs(w, seed=bench.rank_seed(w.seed, rank))
        qs = [torch.empty_like(inp["q"]) for _ in range(world)]
        dist.all_gather(qs, inp["q"].contiguous())
        q.put((rank, red, bool(torch.equal(qs[0], qs[1]))))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_seeding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, red, same_q in res:
        assert red == [11.0, 5.0, 14.0, 300.0, 6.0]
        assert not same_q
