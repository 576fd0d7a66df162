"""GPU parity of pa_swap_blocks (preemption: blocks to CPU RAM and back)
against the oracle's whole-block copies; the decode after a round trip
through pinned host memory is bitwise the decode before it."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, host16

pytestmark = pytest.mark.gpu


def _blocks_of(w, seqs):
    ids = set()
    for s in seqs:
        n = -(-int(w.context_lens[s]) // 16)
        ids.update(int(b) for b in w.block_tables[s, :n])
    return sorted(ids)


def test_swap_out_and_back_in_round_trip():
    w = W.gqa(batch=8)
    d = DeviceStep(w).step()
    before = d.out.clone()
    layers_k = [d.k_cache, d.k_cache.flip(0).contiguous()]       # two layers, different bytes
    layers_v = [d.v_cache, d.v_cache.flip(0).contiguous()]
    blocks = _blocks_of(w, range(4))
    n = len(blocks)
    shape = (n + 3,) + tuple(d.k_cache.shape[1:])
    host_k = [torch.zeros(shape, dtype=d.dt).pin_memory() for _ in range(2)]
    host_v = [torch.zeros(shape, dtype=d.dt).pin_memory() for _ in range(2)]
    out_map = torch.tensor([[b, i] for i, b in enumerate(blocks)], dtype=torch.int64).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.swap_blocks(layers_k, layers_v, host_k, host_v, out_map, dev_error=err)
    torch.cuda.synchronize()
    # oracle on host copies
    ok = [np.zeros((n + 3,) + shape[1:], np.uint16) for _ in range(2)]
    ov = [np.zeros_like(ok[0]) for _ in range(2)]
    oracle.swap_blocks([host16(t) for t in layers_k], [host16(t) for t in layers_v], ok, ov,
                       out_map.cpu().numpy())
    for l in range(2):
        assert np.array_equal(host16(host_k[l]), ok[l])
        assert np.array_equal(host16(host_v[l]), ov[l])

    # the blocks' old ids get reused (poisoned here); swap back in to fresh ids
    # appended to the pool, and remap the tables
    pad = torch.zeros((n,) + tuple(d.k_cache.shape[1:]), dtype=d.dt, device="cuda")
    kc, vc = torch.cat([d.k_cache, pad]), torch.cat([d.v_cache, pad])
    free = list(range(w.num_blocks, w.num_blocks + n))
    for b in blocks:
        kc[b].fill_(float("nan"))
        vc[b].fill_(float("nan"))
    in_map = torch.tensor([[i, f] for i, f in enumerate(free)], dtype=torch.int64).pin_memory()
    pa.swap_blocks(host_k[:1], host_v[:1], [kc], [vc], in_map, dev_error=err)
    remap = dict(zip(blocks, free))
    bt = w.block_tables.copy()
    for s in range(4):
        for j in range(bt.shape[1]):
            if bt[s, j] in remap:
                bt[s, j] = remap[bt[s, j]]
    out2 = torch.empty_like(d.out)
    pa.decode(out2, d.q, kc, vc, torch.from_numpy(bt).cuda(), d.cl, scale=w.scale,
              max_context_len=w.max_context_len, partition_tokens=512)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(before.view(torch.int16), out2.view(torch.int16))


def test_swap_refuses_pageable_host_memory_and_counts_bad_ids():
    w = W.decode_workload("sw", [40, 50], num_q_heads=4, num_kv_heads=2, head_dim=64,
                          dtype="f16", seed=21)
    d = DeviceStep(w).step()
    pageable = torch.zeros((4,) + tuple(d.k_cache.shape[1:]), dtype=d.dt)   # not pinned
    m = torch.tensor([[0, 1]], dtype=torch.int64).cuda()
    with pytest.raises(pa.PaError) as e:
        pa.swap_blocks([d.k_cache], [d.v_cache], [pageable], [pageable.clone()], m)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    host = torch.zeros((4,) + tuple(d.k_cache.shape[1:]), dtype=d.dt).pin_memory()
    host2 = host.clone().pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([[0, 4], [w.num_blocks, 0], [1, 2]], dtype=torch.int64).cuda()
    pa.swap_blocks([d.k_cache], [d.v_cache], [host], [host2], bad, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    assert torch.equal(host[2].view(torch.int16), d.k_cache[1].cpu().view(torch.int16))
    assert (host[0] == 0).all() and (host[1] == 0).all()
