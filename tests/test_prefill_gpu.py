"""GPU parity of pa_prefill_chunk (several query tokens per sequence, causal
within the chunk: chunked prefill, speculative-draft verification) against
the oracle's definition: query token t of a chunk of Tq at the end of an
L-token context is the decode over the first L - Tq + t + 1 tokens."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import (DeviceStep, assert_decode_close, host16, oracle_caches_after_step,
                         to_f64)

pytestmark = pytest.mark.gpu


def _check(w, P=None):
    d = DeviceStep(w, P)
    d.cache_ops()
    d.prefill()
    torch.cuda.synchronize()
    kc, vc = oracle_caches_after_step(w)
    assert np.array_equal(host16(d.k_cache), kc) and np.array_equal(host16(d.v_cache), vc)
    ref = oracle.prefill_chunk(w.q, w.q_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                               w.dtype)
    assert_decode_close(to_f64(d.out), ref, w.name)
    assert int(d.err.item()) == 0
    # with the larger workspace the tcgen05 path runs its work longest first:
    # the same work items, in another order -- the same bits
    alt = d.prefill(torch.full_like(d.out, float("nan")), ordered=True)
    torch.cuda.synchronize()
    assert torch.equal(alt.view(torch.int16), d.out.view(torch.int16)), w.name
    assert int(d.err.item()) == 0
    return d


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2), (16, 1), (12, 1)])
@pytest.mark.parametrize("D,dtype", [(64, "f16"), (128, "bf16")])
def test_ragged_chunks(Hq, Hkv, D, dtype):
    lens = [1, 16, 17, 40, 130, 600, 1100]
    tq = [1, 16, 3, 40, 5, 33, 64]
    w = W.chunk_workload("c", lens, tq, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                         dtype=dtype, seed=Hq * 7 + Hkv + D)
    _check(w)


@pytest.mark.parametrize("P", [0, 16, 128, 512])
def test_chunk_partition_sizes(P):
    w = W.chunk_workload("p", [700, 513, 90, 2000], [100, 9, 90, 4], num_q_heads=8,
                         num_kv_heads=2, head_dim=128, dtype="bf16", seed=P + 3)
    _check(w, P)


def test_spec_verify_and_chunked_prefill_shapes():
    _check(W.spec_verify(batch=12))
    _check(W.chunked_prefill(batch=2, chunk=100))


def test_one_token_chunks_equal_decode_bitwise():
    w = W.decode_workload("one", [5, 200, 700, 1500], num_q_heads=32, num_kv_heads=8,
                          head_dim=128, dtype="bf16", seed=9)
    w.q_start = np.arange(5, dtype=np.int32)
    d = DeviceStep(w)
    d.cache_ops()
    a = d.decode().clone()
    b = d.prefill(torch.empty_like(a))
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bad_query_ranges_are_counted_and_skipped():
    w = W.chunk_workload("bad", [50, 60, 70], [5, 6, 7], num_q_heads=4, num_kv_heads=4,
                         head_dim=64, dtype="f16", seed=4)
    d = DeviceStep(w)
    d.cache_ops()
    qs = torch.from_numpy(w.q_start).cuda()
    qs[2] = 100                         # sequence 1's range runs past the q rows: skipped
    d.out.fill_(5.0)
    pa.prefill_chunk(d.out, d.q, qs, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
                     max_query_len=7, max_context_len=70, partition_tokens=512,
                     dev_error=d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) >= 1
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.prefill_chunk(w.q, w.q_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                               w.dtype)
    out = to_f64(d.out)
    assert_decode_close(out[:5], ref[:5])          # sequence 0 is intact
    assert (out[5:11] == 5.0).all()                # sequence 1 was skipped, nothing written


@pytest.mark.parametrize("scale", [0.0, 1.0])
def test_tensor_core_chunks_scale_zero_and_large_logits(scale):
    """On the tcgen05 path (D 128, many rows): scale 0 makes every row the
    mean of the values it may see; scale 1 with q and K of norm ~11 gives
    logits of tens to hundreds, so the running maximum moves a lot."""
    w = W.chunk_workload("s", [900, 333], [200, 96], num_q_heads=8, num_kv_heads=2,
                         head_dim=128, dtype="bf16", seed=int(scale) + 40)
    w.scale = scale
    _check(w)


@pytest.mark.parametrize("P", [0, 512])
def test_tensor_core_tile_pairs(P):
    """The tcgen05 kernel takes query tiles two at a time: 3, 5 and 9 tiles of
    128 (token, head) rows leave the last pair's second tile empty or partly
    filled, and its rows past the chunk (or in the next sequence) unwritten."""
    w = W.chunk_workload("pairs", [300, 1000, 2500], [96, 160, 288], num_q_heads=8,
                         num_kv_heads=2, head_dim=128, dtype="bf16", seed=50 + P)
    _check(w, P)


@pytest.mark.parametrize("name", ["chunked_prefill", "spec_verify"])
def test_full_size_sampled(name):
    """The two query-chunk workloads at full size, in the launch configuration
    the benchmark times (the chunk workspace, so the tcgen05 path runs its
    longest-first plan): pools bit-exact after the step's writes; outputs on
    sampled rows plus every head of the first and last query token of the
    shortest and the longest sequence."""
    w = W.CONFIGS[name]()
    d = DeviceStep(w)
    d.cache_ops()
    d.prefill(ordered=True)
    torch.cuda.synchronize()
    kc, vc = oracle_caches_after_step(w)
    assert np.array_equal(host16(d.k_cache), kc) and np.array_equal(host16(d.v_cache), vc)
    T, Hq = int(w.q.shape[0]), w.num_q_heads
    rng = np.random.default_rng(31)
    rows = set(rng.choice(T * Hq, size=48, replace=False).tolist())
    for s in (int(np.argmin(w.context_lens)), int(np.argmax(w.context_lens))):
        for tok in (int(w.q_start[s]), int(w.q_start[s + 1]) - 1):
            rows.update(range(tok * Hq, (tok + 1) * Hq))
    rows = np.array(sorted(rows), np.int64)
    ref = oracle.prefill_chunk(w.q, w.q_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                               w.dtype, rows=rows)
    gpu = to_f64(d.out).reshape(T * Hq, -1)[rows]
    assert_decode_close(gpu, ref, name)
    assert int(d.err.item()) == 0


@pytest.mark.parametrize("D,dtype,P", [(128, "bf16", 0), (128, "bf16", 512), (64, "f16", 512)])
def test_bad_table_entry_in_a_chunk_is_skipped_and_counted_once(D, dtype, P):
    """A table entry outside the pool, before the chunk: the block is skipped
    (the tcgen05 path at D 128, the mma.sync path at D 64) and counted once
    however many query tiles read it; the result is the oracle's over the
    table with that entry deleted and the context 16 tokens shorter (the
    order of keys does not matter to attention)."""
    w = W.chunk_workload("badchunk", [900, 1200], [200, 96], num_q_heads=8, num_kv_heads=2,
                         head_dim=D, dtype=dtype, seed=61 + D + P)
    d = DeviceStep(w, P)
    d.cache_ops()
    bt = d.bt.clone()
    bt[0, 10] = w.num_blocks + 7          # tokens 160..175 of sequence 0, before its chunk
    qs = torch.from_numpy(w.q_start).cuda()
    for ordered in (False, True):
        d.err.zero_()
        out = torch.full_like(d.out, float("nan"))
        mq = int(np.diff(w.q_start).max())
        ws = (pa.alloc_chunk_workspace(int(w.q.shape[0]), w.num_seqs, w.num_q_heads,
                                       w.group_size, D, mq, w.max_context_len, P, "cuda")
              if ordered else d.ws)
        pa.prefill_chunk(out, d.q, qs, d.k_cache, d.v_cache, bt, d.cl, scale=w.scale,
                         max_query_len=mq, max_context_len=w.max_context_len,
                         partition_tokens=P, workspace=ws, dev_error=d.err)
        torch.cuda.synchronize()
        assert int(d.err.item()) == 1
        kc, vc = oracle_caches_after_step(w)
        bt_ref = w.block_tables.copy()
        bt_ref[0, 10:-1] = w.block_tables[0, 11:]
        lens = w.context_lens.copy()
        lens[0] -= 16
        ref = oracle.prefill_chunk(w.q, w.q_start, kc, vc, bt_ref, lens, w.scale, w.dtype)
        assert_decode_close(to_f64(out), ref, f"skipped block, ordered={ordered}")


@pytest.mark.parametrize("Hq,Hkv,dtype", [(8, 4, "bf16"), (8, 4, "f16"), (8, 2, "f16"),
                                          (16, 1, "f16"), (4, 4, "f16")])
@pytest.mark.parametrize("P", [0, 256])
def test_tensor_core_groups_and_fp16(Hq, Hkv, dtype, P):
    """The tcgen05 path (D 128, a power-of-two group, enough rows) with fp16
    operands as well as bf16, and at group 2: ragged chunks over several
    partitions, in grid and longest-first order (both checked by _check)."""
    w = W.chunk_workload("tcg", [700, 1500, 260], [120, 64, 260], num_q_heads=Hq,
                         num_kv_heads=Hkv, head_dim=128, dtype=dtype, seed=Hq * 3 + Hkv + P)
    _check(w, P)


@pytest.mark.parametrize("P", [0, 128])
def test_longest_first_chunk_path_over_many_items(P):
    """With the chunk workspace the tcgen05 path runs one CTA per SM, each
    taking (tile pair, partition, KV head) items of the longest-first list from
    a work counter until none is left, its TMEM and barriers carried from item
    to item. 476 items (no split) and 1,542 (128-token partitions) over 148
    SMs: ragged chunks, empty chunks, an empty context, and items whose
    partition lies past their rows' causal limit (no keys: zero partials). The
    result is the grid order's bit for bit and the oracle's within tolerance."""
    rng = np.random.default_rng(77 + P)
    S = 220
    lens = rng.integers(0, 700, size=S)
    tq = np.minimum(lens, rng.integers(0, 72, size=S))
    tq[::17] = 0
    lens[5], tq[5] = 0, 0
    w = W.chunk_workload("many", lens, tq, num_q_heads=8, num_kv_heads=2, head_dim=128,
                         dtype="bf16", seed=78 + P)
    _check(w, P)


def test_argument_errors_on_the_tensor_core_path_counted_once_in_both_orders():
    """Query ranges outside the q rows on the tcgen05 path: each bad sequence
    is counted exactly once (by its first item) and skipped, whether one CTA
    runs one item (grid order) or persistent CTAs take the items from the
    longest-first list; the good sequence's rows are the oracle's."""
    w = W.chunk_workload("badtc", [300, 400, 500], [40, 50, 60], num_q_heads=8, num_kv_heads=2,
                         head_dim=128, dtype="bf16", seed=12)
    d = DeviceStep(w)
    d.cache_ops()
    qs = torch.from_numpy(w.q_start).cuda()
    qs[2] = 10_000          # sequences 1 and 2 now run past the 150 q rows
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.prefill_chunk(w.q, w.q_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                               w.dtype)
    for ordered in (False, True):
        ws = (pa.alloc_chunk_workspace(int(w.q.shape[0]), w.num_seqs, w.num_q_heads,
                                       w.group_size, 128, 60, w.max_context_len, d.P, "cuda")
              if ordered else d.ws)
        d.err.zero_()
        out = torch.full_like(d.out, 5.0)
        pa.prefill_chunk(out, d.q, qs, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
                         max_query_len=60, max_context_len=w.max_context_len,
                         partition_tokens=d.P, workspace=ws, dev_error=d.err)
        torch.cuda.synchronize()
        assert int(d.err.item()) == 2, ordered
        o = to_f64(out)
        assert_decode_close(o[:40], ref[:40], f"good sequence, ordered={ordered}")
        assert (o[40:] == 5.0).all()


def test_tensor_core_output_needs_only_16_byte_alignment():
    """The call asks only for a 16-byte aligned `out`: on the tcgen05 path an
    output view 16 bytes into a buffer (not 32-byte aligned) gets the aligned
    output's bits, in both orders, and nothing is written before the view."""
    w = W.chunk_workload("align", [700, 1500], [120, 64], num_q_heads=8, num_kv_heads=2,
                         head_dim=128, dtype="bf16", seed=91)
    d = DeviceStep(w, 0)
    d.cache_ops()
    for ordered in (False, True):
        a = d.prefill(torch.full_like(d.out, float("nan")), ordered=ordered)
        big = torch.full((d.out.numel() + 8,), float("nan"), dtype=d.out.dtype, device="cuda")
        b = big[8:].view(d.out.shape)
        assert a.data_ptr() % 32 == 0 and b.data_ptr() % 32 == 16
        d.prefill(b, ordered=ordered)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), ordered
        assert torch.isnan(big[:8].float()).all()     # nothing written before the view
    assert int(d.err.item()) == 0
