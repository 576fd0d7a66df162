"""Pins for the fp64 CPU oracle, each against something other than the oracle:
library routines (numpy / torch casts, torch's scaled_dot_product_attention),
closed forms, invariants the pages fix, and hand-written worked examples
from the pages (tests/golden/). No GPU needed.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_391_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(rng, shape, dtype):
    return W._normal_bits(rng, shape, dtype)


def _sdpa(q, K, V, scale):
    """torch's attention in float64: q [Hq, D], K/V [Hkv, L, D] -> [Hq, D]."""
    qt = torch.from_numpy(np.ascontiguousarray(q))[None, :, None, :]
    Kt = torch.from_numpy(np.ascontiguousarray(K))[None]
    Vt = torch.from_numpy(np.ascontiguousarray(V))[None]
    o = F.scaled_dot_product_attention(qt, Kt, Vt, scale=scale,
                                       enable_gqa=K.shape[0] != q.shape[0])
    return o[0, :, 0, :].numpy()


def _paged(contig_k, contig_v, num_blocks, rng, dtype, share=None):
    """Page contiguous per-sequence K/V ([L_s, H_kv, D] bits) into a pool by
    writing every token through oracle.write_kv at the slot its table gives.
    Returns (k_pool, v_pool, block_tables)."""
    S = len(contig_k)
    H, D = contig_k[0].shape[1:]
    alloc = W.ToyBlockAllocator(num_blocks, rng)
    tables = [alloc.allocate(W.blocks_needed(k.shape[0])) for k in contig_k]
    stride = max(1, max(len(t) for t in tables))
    bt = np.full((S, stride), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    nan = W.NAN_BITS[dtype]
    kp = np.full((num_blocks, H, 16, D), nan, dtype=np.uint16)
    vp = np.full_like(kp, nan)
    for s in range(S):
        L = contig_k[s].shape[0]
        slots = np.array([W.slot_of(bt[s], t) for t in range(L)], dtype=np.int64)
        assert oracle.write_kv(contig_k[s], contig_v[s], kp, vp, slots) == 0
    return kp, vp, bt


def _random_case(rng, lens, Hq, Hkv, D, dtype, pool_extra=7):
    ck = [_bits(rng, (L, Hkv, D), dtype) for L in lens]
    cv = [_bits(rng, (L, Hkv, D), dtype) for L in lens]
    q = _bits(rng, (len(lens), Hq, D), dtype)
    nb = sum(W.blocks_needed(L) for L in lens) + pool_extra
    kp, vp, bt = _paged(ck, cv, nb, rng, dtype)
    return q, ck, cv, kp, vp, bt, np.asarray(lens, dtype=np.int32)


# --------------------------------------------------------------------------
# fp16 / bf16 decoding against the library casts, all 65536 patterns
# --------------------------------------------------------------------------

def test_decode16_f16_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.decode16(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_decode16_bf16_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.decode16(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# --------------------------------------------------------------------------
# the pages' worked block-table example (golden fixture)
# --------------------------------------------------------------------------

def _load_block_table_fixture():
    rows, meta = [], {}
    with open(os.path.join(GOLDEN, "block_table_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in ("block_size", "block_table", "context_len"):
                meta[parts[0]] = [int(x) for x in parts[1:]]
            else:
                rows.append([int(x) for x in parts])
    return meta, np.array(rows, dtype=np.int64)


def test_golden_block_table_slots():
    meta, rows = _load_block_table_fixture()
    bt = np.array(meta["block_table"], dtype=np.int32)
    assert meta["block_size"] == [16] and meta["context_len"] == [35]
    assert len(rows) == 35
    assert W.blocks_needed(35) == len(bt)
    for pos, blk, slot, flat in rows:
        assert W.slot_of(bt, int(pos)) == flat


def test_golden_write_places_rows_where_the_example_says():
    """Write 35 distinct rows through the example table and find each one at
    the (physical block, slot) the fixture names; nothing else changes."""
    meta, rows = _load_block_table_fixture()
    bt = np.array(meta["block_table"], dtype=np.int32)
    H, D, NB = 2, 64, 16
    rng = np.random.default_rng(0)
    k = _bits(rng, (35, H, D), "f16")
    v = _bits(rng, (35, H, D), "f16")
    kp = np.full((NB, H, 16, D), 0x7E00, dtype=np.uint16)
    vp = kp.copy()
    before_k = kp.copy()
    assert oracle.write_kv(k, v, kp, vp, rows[:, 3]) == 0
    touched = np.zeros(kp.shape[:1] + kp.shape[2:3], dtype=bool)
    for pos, blk, slot, _ in rows:
        assert np.array_equal(kp[blk, :, slot, :], k[pos])
        assert np.array_equal(vp[blk, :, slot, :], v[pos])
        touched[blk, slot] = True
    untouched = ~touched
    assert np.array_equal(kp.transpose(0, 2, 1, 3)[untouched], before_k.transpose(0, 2, 1, 3)[untouched])
    assert np.array_equal(vp.transpose(0, 2, 1, 3)[untouched], before_k.transpose(0, 2, 1, 3)[untouched])


def test_golden_gather_uses_the_first_L_logical_tokens():
    """With scale 0 every weight is 1/L, so out(L) is the mean of the first L
    logical tokens' values; walking L = 1..35 through the example table pins
    which slot the oracle reads as each logical position."""
    meta, rows = _load_block_table_fixture()
    bt = np.array([meta["block_table"]], dtype=np.int32)
    H, D, NB = 1, 64, 16
    rng = np.random.default_rng(1)
    k = _bits(rng, (35, H, D), "f16")
    v = _bits(rng, (35, H, D), "f16")
    kp = np.full((NB, H, 16, D), 0x7E00, dtype=np.uint16)
    vp = kp.copy()
    oracle.write_kv(k, v, kp, vp, rows[:, 3])
    q = _bits(rng, (1, H, D), "f16")
    vd = oracle.decode16(v, "f16")[:, 0, :]
    for L in range(1, 36):
        out = oracle.decode(q, kp, vp, bt, np.array([L], np.int32), 0.0, "f16")[0, 0]
        np.testing.assert_allclose(out, vd[:L].mean(axis=0), rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# against torch's scaled_dot_product_attention (float64) on contiguous data
# --------------------------------------------------------------------------

@pytest.mark.parametrize("lens,Hq,Hkv,D,dtype", [
    ([8, 17, 34, 51], 4, 4, 64, "f16"),          # the tiny shape
    ([1, 16, 17, 100], 8, 2, 128, "bf16"),        # GQA group 4
    ([33, 300], 16, 2, 128, "bf16"),              # GQA group 8
    ([5, 513, 1030], 2, 2, 128, "f16"),           # spans several 512-token partitions
    ([47], 16, 1, 64, "bf16"),                    # multi-query (group 16)
])
def test_oracle_matches_library_attention(lens, Hq, Hkv, D, dtype):
    rng = np.random.default_rng(sum(lens) + Hq)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, lens, Hq, Hkv, D, dtype)
    scale = 1.0 / np.sqrt(D)
    out = oracle.decode(q, kp, vp, bt, cl, scale, dtype)
    for s, L in enumerate(lens):
        K = oracle.decode16(ck[s], dtype).transpose(1, 0, 2)
        V = oracle.decode16(cv[s], dtype).transpose(1, 0, 2)
        ref = _sdpa(oracle.decode16(q[s], dtype), K, V, scale)
        np.testing.assert_allclose(out[s], ref, rtol=1e-11, atol=1e-12)


def test_wrong_group_mapping_would_be_caught():
    """The library pin distinguishes the contiguous KV-head grouping
    (head h reads KV head h // g) from the interleaved one (h % H_kv)."""
    rng = np.random.default_rng(5)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, [40], 8, 2, 64, "f16")
    out = oracle.decode(q, kp, vp, bt, cl, 0.125, "f16")[0]
    K = oracle.decode16(ck[0], "f16").transpose(1, 0, 2)
    V = oracle.decode16(cv[0], "f16").transpose(1, 0, 2)
    qd = oracle.decode16(q[0], "f16")
    wrong = np.stack([_sdpa(qd[h:h + 1], K[h % 2:h % 2 + 1], V[h % 2:h % 2 + 1], 0.125)[0]
                      for h in range(8)])
    assert np.abs(out - wrong).max() > 1e-2
    np.testing.assert_allclose(out, _sdpa(qd, K, V, 0.125), rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms and special cases
# --------------------------------------------------------------------------

def test_context_len_one_returns_that_value_row():
    rng = np.random.default_rng(2)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, [1, 1, 1], 4, 2, 128, "bf16")
    out = oracle.decode(q, kp, vp, bt, cl, 0.088, "bf16")
    for s in range(3):
        v0 = oracle.decode16(cv[s][0], "bf16")     # [Hkv, D]
        assert np.array_equal(out[s], np.repeat(v0, 2, axis=0))


def test_scale_zero_gives_the_mean_of_values():
    rng = np.random.default_rng(3)
    lens = [3, 16, 40, 129]
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, lens, 2, 2, 64, "f16")
    out = oracle.decode(q, kp, vp, bt, cl, 0.0, "f16")
    for s, L in enumerate(lens):
        mean = oracle.decode16(cv[s], "f16").mean(axis=0)
        np.testing.assert_allclose(out[s], mean, rtol=0, atol=1e-13)


def test_identical_keys_give_uniform_weights():
    rng = np.random.default_rng(4)
    L, H, D = 37, 2, 64
    key = _bits(rng, (1, H, D), "f16")
    ck = [np.repeat(key, L, axis=0)]
    cv = [_bits(rng, (L, H, D), "f16")]
    kp, vp, bt = _paged(ck, cv, 8, rng, "f16")
    q = _bits(rng, (1, H, D), "f16")
    out = oracle.decode(q, kp, vp, bt, np.array([L], np.int32), 0.3, "f16")[0]
    np.testing.assert_allclose(out, oracle.decode16(cv[0], "f16").mean(axis=0), rtol=0, atol=1e-13)


def test_two_token_closed_form():
    """q = a e0, K0 = b e0, K1 = 0: logits scale*a*b and 0, so the weight of
    token 0 is the logistic function of scale*a*b."""
    H, D = 1, 64
    a, b, scale = 2.0, 1.5, 0.25
    q = np.zeros((1, H, D), np.float16); q[0, 0, 0] = a
    k = np.zeros((2, H, D), np.float16); k[0, 0, 0] = b
    rng = np.random.default_rng(6)
    v = _bits(rng, (2, H, D), "f16")
    kp, vp, bt = _paged([k.view(np.uint16)], [v], 4, rng, "f16")
    out = oracle.decode(q.view(np.uint16), kp, vp, bt, np.array([2], np.int32), scale, "f16")[0, 0]
    w0 = 1.0 / (1.0 + np.exp(-scale * a * b))
    vd = oracle.decode16(v, "f16")[:, 0, :]
    np.testing.assert_allclose(out, w0 * vd[0] + (1 - w0) * vd[1], rtol=1e-14, atol=1e-14)


def test_large_logits_do_not_overflow():
    """Logits of several thousand: the softmax must subtract the maximum;
    one key aligned with q dominates and the output is its value row."""
    H, D, L = 1, 64, 20
    rng = np.random.default_rng(7)
    q = np.full((1, H, D), 100.0, np.float16)
    k = np.zeros((L, H, D), np.float16)
    k[11, 0, :] = 60.0   # logit 100*60*64/8 = 48000 ; others 0
    v = _bits(rng, (L, H, D), "f16")
    kp, vp, bt = _paged([k.view(np.uint16)], [v], 4, rng, "f16")
    out = oracle.decode(q.view(np.uint16), kp, vp, bt, np.array([L], np.int32), 1 / 8, "f16")[0, 0]
    assert np.all(np.isfinite(out))
    assert np.array_equal(out, oracle.decode16(v[11, 0], "f16"))


def test_empty_context_gives_zeros():
    rng = np.random.default_rng(8)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, [5, 9], 2, 2, 64, "f16")
    out = oracle.decode(q, kp, vp, bt, np.array([0, 9], np.int32), 0.125, "f16")
    assert np.array_equal(out[0], np.zeros_like(out[0]))
    assert np.all(np.isfinite(out[1]))


# --------------------------------------------------------------------------
# invariants the pages fix
# --------------------------------------------------------------------------

def test_physical_placement_does_not_change_the_result():
    """Logical contiguity does not need physical contiguity ("PagedAttention:
    Decoupling Logical Context ..."): relabelling every physical block gives
    bit-identical output."""
    w = W.tiny()
    kc, vc = w.k_pool.copy(), w.v_pool.copy()
    oracle.copy_blocks([kc], [vc], w.copy_pairs)
    oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping)
    base = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    perm = np.random.default_rng(9).permutation(w.num_blocks)
    kp = np.empty_like(kc); vp = np.empty_like(vc)
    kp[perm] = kc; vp[perm] = vc
    bt = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    out = oracle.decode(w.q, kp, vp, bt, w.context_lens, w.scale, w.dtype)
    assert np.array_equal(base, out)


def test_shared_blocks_equal_private_copies():
    """Sequences whose tables point at the same prefix blocks give the same
    result as sequences holding private byte copies of them."""
    rng = np.random.default_rng(10)
    H, D, P = 2, 128, 48
    prefix_k = _bits(rng, (P, H, D), "bf16")
    prefix_v = _bits(rng, (P, H, D), "bf16")
    kp, vp, bt = _paged([prefix_k], [prefix_v], 64, rng, "bf16")
    shared = bt[0, :3]
    priv = np.array([[40, 41, 42], [50, 51, 52]])
    for row in priv:
        kp[row] = kp[shared]; vp[row] = vp[shared]
    q = _bits(rng, (2, 4, D), "bf16")
    cl = np.array([P, P], np.int32)
    out_shared = oracle.decode(q, kp, vp, np.stack([shared, shared]).astype(np.int32), cl, 0.1, "bf16")
    out_priv = oracle.decode(q, kp, vp, priv.astype(np.int32), cl, 0.1, "bf16")
    assert np.array_equal(out_shared, out_priv)


def _contiguous_from_pool(kp, vp, bt_row, L):
    """Logical-order rows via the (golden-pinned) slot arithmetic."""
    slots = [W.slot_of(bt_row, t) for t in range(L)]
    K = np.stack([kp[s // 16, :, s % 16, :] for s in slots])
    V = np.stack([vp[s // 16, :, s % 16, :] for s in slots])
    return K, V


def test_cow_fork_tiny_step():
    """The tiny step: fork (copy the shared partial block), write one token per
    sequence, decode. Shared full blocks stay byte-identical; each sequence
    sees its own new token; outputs match library attention."""
    w = W.tiny()
    kc, vc = w.k_pool.copy(), w.v_pool.copy()
    shared = w.block_tables[3, :3]
    before = kc[shared].copy(), vc[shared].copy()
    src, dst = w.copy_pairs[0]
    oracle.copy_blocks([kc], [vc], w.copy_pairs)
    assert np.array_equal(kc[dst], kc[src]) and np.array_equal(vc[dst], vc[src])
    oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping)
    assert np.array_equal(kc[shared], before[0]) and np.array_equal(vc[shared], before[1])
    # source and copy now differ exactly in slot 2 (each sequence's own token)
    diff = np.nonzero((kc[src] != kc[dst]).any(axis=(0, 2)))[0]
    assert list(diff) == [2]
    out = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    for s in range(w.num_seqs):
        K, V = _contiguous_from_pool(kc, vc, w.block_tables[s], int(w.context_lens[s]))
        assert not np.isnan(oracle.decode16(K, "f16")).any()
        ref = _sdpa(oracle.decode16(w.q[s], "f16"), oracle.decode16(K, "f16").transpose(1, 0, 2),
                    oracle.decode16(V, "f16").transpose(1, 0, 2), w.scale)
        np.testing.assert_allclose(out[s], ref, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# write_kv / copy_blocks edge cases
# --------------------------------------------------------------------------

def test_write_kv_skips_padding_and_counts_out_of_range():
    rng = np.random.default_rng(11)
    NB, H, D = 4, 2, 64
    kp = np.full((NB, H, 16, D), 0x7E00, np.uint16); vp = kp.copy()
    k = _bits(rng, (4, H, D), "f16"); v = _bits(rng, (4, H, D), "f16")
    slots = np.array([-1, 5, NB * 16, 63], np.int64)
    before = kp.copy()
    assert oracle.write_kv(k, v, kp, vp, slots) == 1
    assert np.array_equal(kp[0, :, 5], k[1]) and np.array_equal(vp[3, :, 15], v[3])
    mask = np.ones((NB, 16), bool); mask[0, 5] = mask[3, 15] = False
    assert np.array_equal(kp.transpose(0, 2, 1, 3)[mask], before.transpose(0, 2, 1, 3)[mask])


def test_copy_blocks_every_layer_and_nothing_else():
    rng = np.random.default_rng(12)
    NB, H, D, nl = 10, 2, 64, 3
    ks = [_bits(rng, (NB, H, 16, D), "bf16") for _ in range(nl)]
    vs = [_bits(rng, (NB, H, 16, D), "bf16") for _ in range(nl)]
    orig_k = [k.copy() for k in ks]; orig_v = [v.copy() for v in vs]
    pairs = np.array([[1, 7], [2, 3], [9, 0]], np.int64)
    oracle.copy_blocks(ks, vs, pairs)
    for l in range(nl):
        for src, dst in pairs:
            assert np.array_equal(ks[l][dst], orig_k[l][src])
            assert np.array_equal(vs[l][dst], orig_v[l][src])
        rest = [b for b in range(NB) if b not in pairs[:, 1]]
        assert np.array_equal(ks[l][rest], orig_k[l][rest])
        assert np.array_equal(vs[l][rest], orig_v[l][rest])


def test_out_of_range_table_entry_is_an_error():
    rng = np.random.default_rng(13)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, [20], 2, 2, 64, "f16")
    bt = bt.copy(); bt[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.decode(q, kp, vp, bt, cl, 0.1, "f16")


def test_rows_subset_matches_full():
    w = W.tiny()
    full = oracle.decode(w.q, w.k_pool, w.v_pool, w.block_tables, w.context_lens - 1, w.scale,
                         w.dtype)
    full[4] = 0  # sequence 4's private block is only filled by the step
    rows = np.array([0, 5, 13, 15], np.int64)
    sub = oracle.decode(w.q[:4], w.k_pool, w.v_pool, w.block_tables[:4], w.context_lens[:4] - 1,
                        w.scale, w.dtype, rows=rows)
    assert np.array_equal(sub, full.reshape(-1, 64)[rows])


def test_swap_blocks_between_pools_of_different_sizes():
    """Swap out (device-sized pool -> small host pool) and back in to other
    block ids: the moved blocks are byte-identical, nothing else changes."""
    rng = np.random.default_rng(14)
    H, D, nl = 2, 64, 2
    dev_k = [_bits(rng, (12, H, 16, D), "bf16") for _ in range(nl)]
    dev_v = [_bits(rng, (12, H, 16, D), "bf16") for _ in range(nl)]
    host_k = [np.zeros((4, H, 16, D), np.uint16) for _ in range(nl)]
    host_v = [np.zeros((4, H, 16, D), np.uint16) for _ in range(nl)]
    orig = [k.copy() for k in dev_k]
    out_pairs = np.array([[3, 0], [9, 1], [4, 2]], np.int64)
    oracle.swap_blocks(dev_k, dev_v, host_k, host_v, out_pairs)
    for l in range(nl):
        for s, d in out_pairs:
            assert np.array_equal(host_k[l][d], dev_k[l][s])
            assert np.array_equal(host_v[l][d], dev_v[l][s])
        assert not host_k[l][3].any()
        assert np.array_equal(dev_k[l], orig[l])          # the source is only read
    in_pairs = np.array([[0, 11], [1, 0], [2, 5]], np.int64)
    oracle.swap_blocks(host_k, host_v, dev_k, dev_v, in_pairs)
    for l in range(nl):
        assert np.array_equal(dev_k[l][11], orig[l][3])
        assert np.array_equal(dev_k[l][0], orig[l][9])
        assert np.array_equal(dev_k[l][5], orig[l][4])
        untouched = [b for b in range(12) if b not in (11, 0, 5)]
        assert np.array_equal(dev_k[l][untouched], orig[l][untouched])


# --------------------------------------------------------------------------
# query chunks (chunked prefill / speculative verification)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("lens,tq,Hq,Hkv,D,dtype", [
    ([20, 5, 40], [3, 5, 1], 4, 2, 64, "f16"),
    ([100, 37], [17, 4], 8, 2, 128, "bf16"),
    ([64], [64], 2, 1, 64, "f16"),                 # the whole context is the chunk
])
def test_prefill_chunk_matches_library_attention_with_causal_mask(lens, tq, Hq, Hkv, D, dtype):
    """Query token t of a chunk of Tq at the end of an L-token context sees
    keys 0 .. L-Tq+t: torch's attention with that (bottom-right aligned)
    boolean mask on the contiguous context."""
    rng = np.random.default_rng(sum(lens) + sum(tq))
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, lens, Hq, Hkv, D, dtype)
    q_start = np.concatenate([[0], np.cumsum(tq)]).astype(np.int32)
    qc = _bits(rng, (int(q_start[-1]), Hq, D), dtype)
    scale = 1 / np.sqrt(D)
    out = oracle.prefill_chunk(qc, q_start, kp, vp, bt, cl, scale, dtype)
    for s, (L, T) in enumerate(zip(lens, tq)):
        K = torch.from_numpy(oracle.decode16(ck[s], dtype).transpose(1, 0, 2))[None]
        V = torch.from_numpy(oracle.decode16(cv[s], dtype).transpose(1, 0, 2))[None]
        Q = torch.from_numpy(oracle.decode16(qc[q_start[s]:q_start[s + 1]], dtype).transpose(1, 0, 2))[None]
        pos_q = torch.arange(L - T, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos_q           # [T, L]
        ref = F.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale,
                                             enable_gqa=Hkv != Hq)[0].transpose(0, 1).numpy()
        np.testing.assert_allclose(out[q_start[s]:q_start[s + 1]], ref, rtol=1e-11, atol=1e-12)
        if T == L:   # a chunk that is the whole context is ordinary causal attention
            ref2 = F.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=scale,
                                                  enable_gqa=Hkv != Hq)[0].transpose(0, 1).numpy()
            np.testing.assert_allclose(out[q_start[s]:q_start[s + 1]], ref2, rtol=1e-11, atol=1e-12)


def test_one_token_chunks_are_decode():
    rng = np.random.default_rng(15)
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, [9, 30, 77], 4, 2, 64, "bf16")
    q_start = np.arange(4, dtype=np.int32)
    a = oracle.prefill_chunk(q, q_start, kp, vp, bt, cl, 0.125, "bf16")
    b = oracle.decode(q, kp, vp, bt, cl, 0.125, "bf16")
    assert np.array_equal(a, b)


def test_prefill_chunk_scale_zero_is_the_running_mean_of_values():
    """Closed form: with scale 0 every visible key weighs the same, so query
    token t of a chunk of Tq at the end of an L-token context returns the mean
    of V over positions 0 .. L-Tq+t (a prefix mean that grows by one key per
    query token)."""
    rng = np.random.default_rng(77)
    lens, tq, Hq, Hkv, D = [12, 33], [5, 33], 4, 2, 64
    q, ck, cv, kp, vp, bt, cl = _random_case(rng, lens, Hq, Hkv, D, "f16")
    q_start = np.concatenate([[0], np.cumsum(tq)]).astype(np.int32)
    qc = _bits(rng, (int(q_start[-1]), Hq, D), "f16")
    out = oracle.prefill_chunk(qc, q_start, kp, vp, bt, cl, 0.0, "f16")
    for s, (L, T) in enumerate(zip(lens, tq)):
        V = oracle.decode16(cv[s], "f16")                   # [L, Hkv, D]
        for t in range(T):
            n = L - T + t + 1
            mean = V[:n].mean(axis=0)                       # [Hkv, D]
            want = np.repeat(mean, Hq // Hkv, axis=0)       # query head h -> KV head h // g
            np.testing.assert_allclose(out[q_start[s] + t], want, rtol=1e-12, atol=1e-13)
