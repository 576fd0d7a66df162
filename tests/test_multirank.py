"""The multi-GPU bookkeeping of bench.py on CPU: world size 2 over gloo.

Each rank runs an independent workload (weak scaling); the only collectives
are the timing reduction (max of times, sum of work). Here the ranks hand in
different numbers and must agree on the same whole-job figures.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import datetime

    import torch.distributed as dist

    import bench
    from paged_kv_cache_391_b200 import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.make_workload("gqa", 4, seed_offset=rank)
        res = {"w": w, "elapsed_ms": 10.0 + 5.0 * rank, "e2e": {"ms": 20.0 - rank},
               "att_ms": 1.0 + rank, "write_ms": 0.5 - 0.1 * rank, "copy_ms": None,
               "errors": rank}
        agg = bench.reduce_over_ranks(res, world, device=None)
        q.put((rank, agg, w.kv_bytes(), int(w.context_lens.sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_agree_on_whole_job_figures():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    (r0, a0, kv0, t0), (r1, a1, kv1, t1) = res
    assert a0 == a1                                   # every rank sees the same figures
    assert a0["ms"] == 15.0 and a0["e2e_ms"] == 20.0  # slowest rank
    assert a0["att_ms"] == 2.0 and a0["write_ms"] == 0.5 and a0["copy_ms"] is None
    assert a0["kv"] == kv0 + kv1 and a0["seqs"] == 8 and a0["errors"] == 1
    assert t0 != t1                                   # ranks ran different (independent) workloads


def test_single_rank_is_the_identity():
    import bench
    from paged_kv_cache_391_b200 import workloads as W
    w = W.tiny()
    res = {"w": w, "elapsed_ms": 3.0, "e2e": None, "att_ms": 2.5, "write_ms": 0.25,
           "copy_ms": 0.125, "errors": 0}
    agg = bench.reduce_over_ranks(res, 1)
    assert agg == {"ms": 3.0, "e2e_ms": 0.0, "att_ms": 2.5, "write_ms": 0.25, "copy_ms": 0.125,
                   "sus_ms": 0.0, "kv": float(w.kv_bytes()), "seqs": 5.0, "errors": 0}


def _shard_worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank: its own shard of sequences, decoded with no exchange
        w = bench.make_workload("gqa", 3, seed_offset=rank)
        kc, vc = w.k_pool.copy(), w.v_pool.copy()
        oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping)
        out = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
        got = [torch.zeros(out.size, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(np.ascontiguousarray(out).reshape(-1)))
        if rank == 0:
            q.put([g.numpy() for g in got])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_sequence_shards_need_no_exchange():
    """The data-parallel split: each rank decodes its own sequences; the
    whole job's output is the concatenation of the ranks' outputs, each equal
    to a single process decoding that shard, and the shards differ."""
    import numpy as np

    import bench
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    gathered = q.get()          # before joining: the result does not fit in the pipe's buffer
    for p in procs:
        p.join(200)
        assert p.exitcode == 0
    for r in range(world):
        w = bench.make_workload("gqa", 3, seed_offset=r)
        kc, vc = w.k_pool.copy(), w.v_pool.copy()
        oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping)
        want = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
        assert np.array_equal(gathered[r], want.reshape(-1))
    assert not np.array_equal(gathered[0], gathered[1])
