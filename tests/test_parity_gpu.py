"""GPU parity: libpa's kernels (through the C ABI) against the fp64 oracle.

write_kv and copy_blocks must match bit for bit over the whole pool (NaN
fill included); decode must be within max-abs 2e-2 and per-row relative
1e-2 of the oracle. Sizes span several 16-token tiles, several 512-token
partitions and ragged tails; edge cases cover empty and one-token contexts,
partition sizes, every supported group size, head dim and dtype.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import (DeviceStep, assert_decode_close, dev16, host16, oracle_caches_after_step,
                         to_f64, torch_dtype)

pytestmark = pytest.mark.gpu


def _full_check(w, partition_tokens=None):
    d = DeviceStep(w, partition_tokens).step()
    kc, vc = oracle_caches_after_step(w)
    assert np.array_equal(host16(d.k_cache), kc), "k_cache differs from the oracle"
    assert np.array_equal(host16(d.v_cache), vc), "v_cache differs from the oracle"
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    assert_decode_close(to_f64(d.out), ref, w.name)
    assert int(d.err.item()) == 0
    return d, ref


# ------------------------------------------------------------ the five shapes, small sizes

def test_tiny_step():
    _full_check(W.tiny())


@pytest.mark.parametrize("make", [
    lambda: W.mha(batch=4),
    lambda: W.gqa(batch=12),
    lambda: W.shared_prefix(num_seqs=4, prefix=700, suffix_hi=100),
    lambda: W.long_context(batch=2, lo=3000, hi=6000),
], ids=["mha", "gqa", "shared_prefix", "long"])
def test_scaled_down_configs(make):
    _full_check(make())


@pytest.mark.parametrize("P", [0, 16, 64, 512, 2048])
def test_partition_sizes_agree(P):
    w = W.decode_workload("p", [1, 15, 16, 17, 511, 512, 513, 1024, 1500, 2100],
                          num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="bf16", seed=P + 1)
    _full_check(w, partition_tokens=P)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (16, 2), (16, 1), (12, 1), (6, 2)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_group_sizes_head_dims_dtypes(Hq, Hkv, D, dtype):
    w = W.decode_workload("g", [3, 40, 700], num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          dtype=dtype, seed=Hq * 100 + Hkv * 10 + D)
    _full_check(w)


# ------------------------------------------------------------ special cases

def test_context_len_one_returns_the_value_row_exactly():
    w = W.decode_workload("one", [1, 1, 1], num_q_heads=8, num_kv_heads=2, head_dim=128,
                          dtype="bf16", seed=3)
    d = DeviceStep(w).step()
    # the token at position 0 is the new token of this step
    v0 = w.new_v  # [S, Hkv, D]
    want = np.repeat(v0, 4, axis=1)
    assert np.array_equal(host16(d.out), want)


def test_empty_context_gives_zeros():
    w = W.decode_workload("e", [5, 40], num_q_heads=4, num_kv_heads=4, head_dim=64, dtype="f16",
                          seed=4)
    d = DeviceStep(w)
    d.cache_ops()
    d.cl.copy_(torch.tensor([0, 40], dtype=torch.int32))
    d.decode()
    torch.cuda.synchronize()
    out = to_f64(d.out)
    assert (out[0] == 0).all() and np.isfinite(out[1]).all()


def test_all_empty_contexts():
    w = W.decode_workload("e0", [1, 1], num_q_heads=4, num_kv_heads=4, head_dim=64, dtype="f16",
                          seed=5)
    d = DeviceStep(w)
    d.cl.zero_()
    d.out.fill_(7.0)
    pa.decode(d.out, d.q, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale, max_context_len=0,
              partition_tokens=512)
    torch.cuda.synchronize()
    assert (to_f64(d.out) == 0).all()


def test_identical_keys_give_the_mean_of_values():
    rng = np.random.default_rng(6)
    w = W.decode_workload("same", [77], num_q_heads=4, num_kv_heads=1, head_dim=128, dtype="bf16",
                          seed=6)
    kp = w.k_pool.copy()
    key = kp[w.block_tables[0, 0], 0, 0].copy()
    kp[:, :, :, :] = key
    w.k_pool = kp
    w.new_k[:] = key
    d = DeviceStep(w).step()
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    assert_decode_close(to_f64(d.out), ref)


def test_physical_permutation_is_bitwise_invariant():
    w = W.gqa(batch=6)
    d1 = DeviceStep(w).step()
    perm = np.random.default_rng(7).permutation(w.num_blocks)
    kp = np.empty_like(w.k_pool); vp = np.empty_like(w.v_pool)
    kp[perm] = w.k_pool; vp[perm] = w.v_pool
    w2 = W.DecodeWorkload(**{**w.__dict__})
    w2.k_pool, w2.v_pool = kp, vp
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)],
                               -1).astype(np.int32)
    w2.slot_mapping = (perm[w.slot_mapping // 16] * 16 + w.slot_mapping % 16).astype(np.int64)
    d2 = DeviceStep(w2).step()
    assert torch.equal(d1.out.view(torch.int16), d2.out.view(torch.int16))


def test_shared_blocks_equal_private_copies_bitwise():
    w = W.shared_prefix(num_seqs=3, prefix=600, suffix_hi=60)
    d = DeviceStep(w).step()
    # give every sequence private copies of the shared full prefix blocks
    full = 600 // 16
    extra = 2 * full
    pad = torch.zeros((extra,) + tuple(d.k_cache.shape[1:]), dtype=d.dt, device="cuda")
    kc, vc = torch.cat([d.k_cache, pad]), torch.cat([d.v_cache, pad])
    free = list(range(w.num_blocks, w.num_blocks + extra))
    bt = w.block_tables.copy()
    for s in range(1, 3):
        for j in range(full):
            nb = free.pop()
            kc[nb] = kc[bt[s, j]]
            vc[nb] = vc[bt[s, j]]
            bt[s, j] = nb
    out2 = torch.empty_like(d.out)
    pa.decode(out2, d.q, kc, vc, torch.from_numpy(bt).cuda(), d.cl, scale=w.scale,
              max_context_len=w.max_context_len, partition_tokens=512)
    torch.cuda.synchronize()
    assert torch.equal(d.out.view(torch.int16), out2.view(torch.int16))


def test_repeated_runs_are_bitwise_identical():
    w = W.long_context(batch=2, lo=2000, hi=4000)
    d = DeviceStep(w).step()
    first = d.out.clone()
    for _ in range(3):
        d.decode()
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), d.out.view(torch.int16))


def test_split_matches_unsplit():
    w = W.long_context(batch=2, lo=3000, hi=5000)
    a = DeviceStep(w, partition_tokens=512).step()
    b = DeviceStep(w, partition_tokens=0).step()
    assert_decode_close(to_f64(a.out), to_f64(b.out), "split vs unsplit")


def test_no_write_outside_the_output():
    """Canary regions before and after the output stay untouched."""
    w = W.gqa(batch=5)
    d = DeviceStep(w)
    d.cache_ops()
    n = d.out.numel()
    buf = torch.full((n + 2048,), 3.0, dtype=d.dt, device="cuda")
    out = buf[1024:1024 + n].view(d.out.shape)
    d.decode(out)
    torch.cuda.synchronize()
    assert (buf[:1024] == 3.0).all() and (buf[1024 + n:] == 3.0).all()
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    assert_decode_close(to_f64(out), ref)


# ------------------------------------------------------------ device-data violations

def test_write_kv_out_of_range_slot_is_counted_and_skipped():
    w = W.decode_workload("bad", [10, 20, 30], num_q_heads=4, num_kv_heads=2, head_dim=64,
                          dtype="f16", seed=8)
    d = DeviceStep(w)
    slots = d.slots.clone()
    slots[1] = w.num_blocks * 16 + 3
    slots[2] = -1
    pa.write_kv(d.new_k, d.new_v, d.k_cache, d.v_cache, slots, dev_error=d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 1
    kc, vc = w.k_pool.copy(), w.v_pool.copy()
    oracle.write_kv(w.new_k[:1], w.new_v[:1], kc, vc, w.slot_mapping[:1])
    assert np.array_equal(host16(d.k_cache), kc) and np.array_equal(host16(d.v_cache), vc)


def test_decode_bad_table_entry_is_counted_and_skipped():
    w = W.decode_workload("badbt", [40, 40], num_q_heads=8, num_kv_heads=2, head_dim=128,
                          dtype="bf16", seed=9)
    d = DeviceStep(w)
    d.cache_ops()
    bt = d.bt.clone()
    bt[0, 1] = w.num_blocks + 5
    pa.decode(d.out, d.q, d.k_cache, d.v_cache, bt, d.cl, scale=w.scale, max_context_len=40,
              partition_tokens=512, dev_error=d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 1     # counted once (by the KV-head-0 CTA)
    out = to_f64(d.out)
    assert np.isfinite(out).all()
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    assert_decode_close(out[1], ref[1])
    # skipping a full block is attention over the other tokens, and attention
    # does not depend on the order of its keys: the oracle over the table with
    # that entry deleted and the context 16 tokens shorter
    bt0 = np.delete(w.block_tables[0], 1)[None, :]
    ref0 = oracle.decode(w.q[:1], kc, vc, bt0, np.array([24], np.int32), w.scale, w.dtype)
    assert_decode_close(out[:1], ref0, "skipped block")


def test_context_longer_than_max_is_clamped_and_counted():
    w = W.decode_workload("clamp", [100, 60], num_q_heads=4, num_kv_heads=4, head_dim=64,
                          dtype="f16", seed=10)
    d = DeviceStep(w)
    d.cache_ops()
    pa.decode(d.out, d.q, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale, max_context_len=80,
              partition_tokens=32, dev_error=d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 1
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, np.array([80, 60], np.int32), w.scale, w.dtype)
    assert_decode_close(to_f64(d.out), ref)


def test_copy_blocks_multi_layer_bit_exact():
    rng = np.random.default_rng(11)
    NB, H, D, nl = 20, 8, 128, 3
    ks = [W._normal_bits(rng, (NB, H, 16, D), "bf16") for _ in range(nl)]
    vs = [W._normal_bits(rng, (NB, H, 16, D), "bf16") for _ in range(nl)]
    pairs = np.array([[1, 7], [2, 3], [19, 0], [5, 6]], np.int64)
    dk = [dev16(k, torch.bfloat16) for k in ks]
    dv = [dev16(v, torch.bfloat16) for v in vs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.copy_blocks(dk, dv, torch.from_numpy(pairs).cuda(), dev_error=err)
    bad = torch.tensor([[0, NB]], dtype=torch.int64, device="cuda")
    pa.copy_blocks(dk, dv, bad, dev_error=err)
    torch.cuda.synchronize()
    oracle.copy_blocks(ks, vs, pairs)
    assert int(err.item()) == 1
    for l in range(nl):
        assert np.array_equal(host16(dk[l]), ks[l]) and np.array_equal(host16(dv[l]), vs[l])


# ------------------------------------------------------------ full sizes, bench launch config

FULL = {
    "mha": lambda: W.mha(),
    "gqa": lambda: W.gqa(),
    "shared_prefix": lambda: W.shared_prefix(),
    "long": lambda: W.long_context(),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled(name):
    """Full-size configs as the benchmark runs them: whole pools bit-exact after
    the step; decode checked on sampled rows plus every head of the shortest
    and the longest sequence."""
    w = FULL[name]()
    d = DeviceStep(w).step()
    kc, vc = oracle_caches_after_step(w)
    assert np.array_equal(host16(d.k_cache), kc)
    assert np.array_equal(host16(d.v_cache), vc)
    S, Hq = w.num_seqs, w.num_q_heads
    rng = np.random.default_rng(12)
    rows = set(rng.choice(S * Hq, size=min(48, S * Hq), replace=False).tolist())
    for s in (int(np.argmin(w.context_lens)), int(np.argmax(w.context_lens))):
        rows.update(range(s * Hq, (s + 1) * Hq))
    rows = np.array(sorted(rows), np.int64)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype, rows=rows)
    gpu = to_f64(d.out).reshape(S * Hq, -1)[rows]
    assert_decode_close(gpu, ref, name)
    assert int(d.err.item()) == 0
