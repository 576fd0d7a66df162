"""The input generator: the pages' worked numbers (tests/golden/page_arithmetic.txt)
and the structure of the five named configurations. No GPU needed."""
import os

import numpy as np
import pytest

import oracle
from paged_kv_cache_391_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _arith():
    rows = []
    with open(os.path.join(GOLDEN, "page_arithmetic.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, *vals = line.split()
                rows.append((k, [float(v) for v in vals]))
    return rows


@pytest.mark.parametrize("key,vals", _arith())
def test_page_arithmetic(key, vals):
    if key == "tokens_to_blocks":
        assert W.blocks_needed(int(vals[0])) == int(vals[1])
    elif key == "free_slots_in_last_block":
        n = int(vals[0])
        assert W.blocks_needed(n) * 16 - n == int(vals[1])
    elif key == "unshared_tokens":
        assert int(vals[0]) * int(vals[1]) == int(vals[2])
    elif key == "reserved":
        assert int(vals[0]) * int(vals[1]) == int(vals[2])
    elif key == "used":
        assert sum(int(v) for v in vals[:-1]) == int(vals[-1])
    elif key == "utilisation_percent":
        assert round(100 * vals[0] / vals[1]) == int(vals[2])
    elif key == "kv_bytes_per_token":
        L, H, D, b, want = (int(v) for v in vals)
        assert W.kv_cache_bytes(L, H, D, 1, b) == want
    elif key == "kv_gib_at_tokens":
        L, H, D, b, T = (int(v) for v in vals[:5])
        assert W.kv_cache_bytes(L, H, D, T, b) / 2**30 == pytest.approx(vals[5], rel=1e-12)
    elif key == "mean_last_block_waste":
        bs = int(vals[0])
        # every fill 1..bs of the last block equally likely
        waste = np.mean([W.blocks_needed(n) * bs - n for n in range(1, bs + 1)])
        assert waste == pytest.approx(vals[1])
    else:
        raise AssertionError(key)


def test_waste_on_uniform_lengths_is_about_half_a_block():
    """The mha lengths (uniform in [128, 2048]) waste ~7.5 slots per sequence."""
    w = W.mha(batch=64)
    waste = np.array([W.blocks_needed(L) * 16 - L for L in w.context_lens])
    assert 5.0 < waste.mean() < 10.0
    assert (waste >= 0).all() and (waste < 16).all()


def test_allocator_scatters_and_never_reuses():
    rng = np.random.default_rng(0)
    a = W.ToyBlockAllocator(100, rng)
    got = np.concatenate([a.allocate(10) for _ in range(10)])
    assert sorted(got.tolist()) == list(range(100))
    assert not np.all(np.diff(got) == 1)
    with pytest.raises(MemoryError):
        a.allocate(1)


def test_tiny_structure():
    w = W.tiny()
    assert w.context_lens.tolist() == [8, 17, 34, 51, 51]
    assert w.num_blocks == 32 and w.head_dim == 64 and w.dtype == "f16"
    # the fork shares sequence 3's three full blocks and owns a copy of the 4th
    assert np.array_equal(w.block_tables[4, :3], w.block_tables[3, :3])
    src, dst = w.copy_pairs[0]
    assert src == w.block_tables[3, 3] and dst == w.block_tables[4, 3]
    # every table entry within a context is a distinct block except the shared ones
    used = [w.block_tables[s, :W.blocks_needed(L)] for s, L in enumerate(w.context_lens)]
    flat = np.concatenate(used)
    assert len(set(flat.tolist())) == len(flat) - 3
    # each sequence writes position context_len - 1
    for s in range(5):
        assert w.slot_mapping[s] == W.slot_of(w.block_tables[s], int(w.context_lens[s]) - 1)


def _after_step(w):
    kc, vc = w.k_pool.copy(), w.v_pool.copy()
    if len(w.copy_pairs):
        oracle.copy_blocks([kc], [vc], w.copy_pairs)
    assert oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping) == 0
    return kc, vc


@pytest.mark.parametrize("make", [
    lambda: W.tiny(),
    lambda: W.mha(batch=3),
    lambda: W.gqa(batch=5),
    lambda: W.shared_prefix(num_seqs=3, prefix=200, suffix_hi=40),
    lambda: W.long_context(batch=1, lo=1100, hi=1500),
])
def test_every_attended_slot_holds_a_token_after_the_step(make):
    """After the step's copies and writes, every slot inside a context holds a
    number and the decode over it is finite; slots outside stay NaN."""
    w = make()
    kc, vc = _after_step(w)
    nan = W.NAN_BITS[w.dtype]
    for s, L in enumerate(w.context_lens):
        for t in range(int(L)):
            slot = W.slot_of(w.block_tables[s], t)
            assert (kc[slot // 16, :, slot % 16] != nan).all()
            assert (vc[slot // 16, :, slot % 16] != nan).all()
    out = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    assert np.isfinite(out).all()


def test_shared_prefix_structure():
    """The step of the shared-prefix config: the prefix's 312 full blocks are
    shared, each sequence already owns a copy of the partial prefix block
    (its first 8 slots are the shared block's bits, as the fork's copy left
    them) and its suffix up to the newest token; the step writes one token
    per sequence and copies nothing."""
    w = W.shared_prefix(num_seqs=4, prefix=5000, suffix_hi=40)
    full = 5000 // 16
    assert full == 312 and W.blocks_needed(5000) == 313
    for s in range(1, 4):
        assert np.array_equal(w.block_tables[s, :full], w.block_tables[0, :full])
    assert len(w.copy_pairs) == 0
    forks = np.asarray(w.notes["fork_pairs"])
    assert forks.shape == (4, 2)
    assert (forks[:, 0] == w.notes["partial_prefix_block"]).all()
    assert len(set(forks[:, 1].tolist())) == 4
    assert (forks[:, 1] == w.block_tables[:, full]).all()
    src = w.notes["partial_prefix_block"]
    for dst in forks[:, 1]:
        assert np.array_equal(w.k_pool[dst, :, :8], w.k_pool[src, :, :8])
        assert np.array_equal(w.v_pool[dst, :, :8], w.v_pool[src, :, :8])
    assert w.slot_mapping.size == 4
    for s in range(4):
        assert w.slot_mapping[s] == W.slot_of(w.block_tables[s], int(w.context_lens[s]) - 1)


def test_config_shapes():
    w = W.gqa(batch=16)
    assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.dtype) == (32, 8, 128, "bf16")
    assert (w.context_lens >= 16).all() and (w.context_lens <= 8192).all()
    w = W.long_context(batch=2, lo=2000, hi=3000)
    assert (w.num_q_heads, w.num_kv_heads, w.partition_tokens) == (64, 8, 512)
    w = W.mha(batch=8)
    assert (w.num_q_heads, w.num_kv_heads, w.dtype) == (32, 32, "f16")
    assert (w.context_lens >= 128).all() and (w.context_lens <= 2048).all()
    assert w.num_blocks == int(np.ceil(1.5 * sum(W.blocks_needed(L) for L in w.context_lens)))


def test_seeded_reproducible():
    a, b = W.tiny(), W.tiny()
    for f in ("k_pool", "v_pool", "q", "new_k", "block_tables", "slot_mapping"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


def test_skewed_structure():
    w = W.skewed(batch=40, n_long=3, long_lo=2000, long_hi=3000, short_median=100,
                 short_hi=500)
    lens = w.context_lens
    assert w.num_seqs == 40 and (w.num_q_heads, w.num_kv_heads, w.head_dim) == (32, 8, 128)
    assert int((lens >= 2000).sum()) == 3 and lens.max() <= 3000
    short = lens[lens < 2000]
    assert short.min() >= 16 and short.max() <= 500
    assert w.max_context_len == lens.max()
