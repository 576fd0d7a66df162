"""GPU parity of pa_decode_persistent, the work-queue schedule of decode.

Each (sequence, partition, KV head) item is computed exactly as pa_decode
computes it, so the two must agree bit for bit at the same partition size;
the persistent result is also held to the oracle's tolerance. Cases cover
skewed lengths (a few long contexts among short ones), many more items than
resident CTAs (ring phases carried across items), empty and one-token
contexts, every group size path, both head dims and dtypes, repeated calls on
one workspace, and the host-side error counts (bad table entries, lengths
past max_context_len) matching pa_decode's.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, assert_decode_close, host16, oracle_caches_after_step, to_f64

pytestmark = pytest.mark.gpu


def _persistent(d, out=None, partition_tokens=None, ws=None):
    w = d.w
    P = d.P if partition_tokens is None else partition_tokens
    # NaN everywhere a missing item would leave its mark: the output and
    # the partials the reduce reads
    out = torch.full_like(d.out, float("nan")) if out is None else out
    if ws is None:
        ws = pa.alloc_workspace(int(w.q.shape[0]), w.num_q_heads, w.head_dim, w.max_context_len,
                                P, "cuda", persistent=True)
        ws.fill_(0xFF)
    pa.decode(out, d.q, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
              max_context_len=w.max_context_len, partition_tokens=P, workspace=ws,
              dev_error=d.err, persistent=True)
    torch.cuda.synchronize()
    return out


def _check(w, partition_tokens=None, seqs=None):
    """Bitwise equality with pa_decode, then the oracle's tolerance (on every
    head of the sequences ``seqs`` only, when given)."""
    d = DeviceStep(w, partition_tokens).step()
    got = _persistent(d)
    assert torch.equal(got.view(torch.int16), d.out.view(torch.int16)), \
        f"{w.name}: persistent schedule differs from pa_decode"
    kc, vc = oracle_caches_after_step(w)
    if seqs is None:
        ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
        assert_decode_close(to_f64(got), ref, w.name)
    else:
        Hq, D = w.num_q_heads, w.head_dim
        flat = (np.asarray(seqs)[:, None] * Hq + np.arange(Hq)[None, :]).reshape(-1)
        ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype,
                            rows=flat)
        assert_decode_close(to_f64(got).reshape(-1, D)[flat], ref, w.name)
    assert int(d.err.item()) == 0
    return d, got


@pytest.mark.parametrize("make", [
    W.tiny,
    lambda: W.mha(batch=4),
    lambda: W.gqa(batch=12),
    lambda: W.shared_prefix(num_seqs=4, prefix=700, suffix_hi=100),
    lambda: W.long_context(batch=2, lo=3000, hi=6000),
], ids=["tiny", "mha", "gqa", "shared_prefix", "long"])
def test_scaled_down_configs(make):
    _check(make())


def test_skewed_lengths():
    """A few long contexts among many short ones: most of the grid pa_decode
    launches is empty partitions; the work list holds only the real ones."""
    w = W.skewed(batch=48, n_long=3, long_lo=6000, long_hi=12000, short_median=200,
                 short_hi=1500)
    _check(w)


@pytest.mark.parametrize("P", [0, 16, 64, 512, 2048])
def test_partition_sizes(P):
    w = W.decode_workload("p", [1, 15, 16, 17, 511, 512, 513, 1024, 1500, 2100],
                          num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="bf16", seed=P + 7)
    _check(w, partition_tokens=P)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 1), (12, 1)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_group_sizes_head_dims_dtypes(Hq, Hkv, D, dtype):
    w = W.decode_workload("g", [3, 40, 700, 1300], num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          dtype=dtype, seed=Hq * 100 + Hkv * 10 + D + 1)
    _check(w)


def test_many_items_per_cta():
    """2000 sequences x 8 KV heads with 1..150 tokens: each resident CTA takes
    dozens of items whose tile counts per warp differ (0 to 3), so the ring's
    stage and parity must carry across items."""
    rng = np.random.default_rng(11)
    lens = rng.integers(1, 150, size=2000, endpoint=True)
    w = W.decode_workload("many", lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                          dtype="bf16", seed=11, partition_tokens=64)
    seqs = np.unique(np.concatenate([np.arange(8), rng.choice(2000, size=120, replace=False),
                                     np.arange(1992, 2000)]))
    _check(w, seqs=seqs)


def test_empty_contexts_and_all_empty():
    w = W.decode_workload("e", [0, 5, 0, 600, 0], num_q_heads=8, num_kv_heads=2, head_dim=64,
                          dtype="f16", seed=21)
    d, got = _check(w)
    z = host16(got)[[0, 2, 4]]
    assert not z.any(), "an empty context must give zeros"
    w0 = W.decode_workload("e0", [0, 0, 0], num_q_heads=4, num_kv_heads=4, head_dim=128,
                           dtype="bf16", seed=22)
    _, got0 = _check(w0)
    assert not host16(got0).any()


def test_repeated_calls_reuse_one_workspace():
    w = W.gqa(batch=24)
    d = DeviceStep(w).step()
    ws = pa.alloc_workspace(24, w.num_q_heads, w.head_dim, w.max_context_len, d.P, "cuda",
                            persistent=True)
    a = _persistent(d, ws=ws)
    for _ in range(3):
        b = _persistent(d, ws=ws)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), d.out.view(torch.int16))


def test_error_counts_match_pa_decode():
    """A table entry outside the pool and a length past max_context_len are
    counted (once per sequence / per bad entry, as pa_decode counts them) and
    give pa_decode's output."""
    w = W.decode_workload("bad", [40, 700, 1200], num_q_heads=8, num_kv_heads=2, head_dim=128,
                          dtype="bf16", seed=31)
    d = DeviceStep(w).step()
    bt = d.bt.clone()
    bt[1, 3] = w.k_pool.shape[0] + 5      # outside the pool
    cl = d.cl.clone()
    cl[2] = w.max_context_len + 100       # past max_context_len: clamped
    outs, errs = [], []
    for persistent in (False, True):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.empty_like(d.out)
        pa.decode(out, d.q, d.k_cache, d.v_cache, bt, cl, scale=w.scale,
                  max_context_len=w.max_context_len, partition_tokens=d.P, dev_error=err,
                  persistent=persistent)
        torch.cuda.synchronize()
        outs.append(out)
        errs.append(int(err.item()))
    assert errs[0] == errs[1] and errs[0] > 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_full_size_skewed_sampled_rows():
    """The benchmark's skewed batch (256 sequences, 4 of 64k-128k tokens) at
    full size, in the launch configuration the benchmark times: bitwise equal
    to pa_decode everywhere, sampled rows (every long one) against the oracle."""
    w = W.skewed()
    long_seqs = np.flatnonzero(w.context_lens > 10000)
    rng = np.random.default_rng(5)
    seqs = np.unique(np.concatenate([long_seqs, rng.choice(256, size=12, replace=False)]))
    _check(w, seqs=seqs)


def test_plan_lists_every_item_once_longest_first():
    """White-box check of the work list the plan kernel leaves in the
    workspace (after pa_decode's partials: num_seqs * partitions 32-bit items
    (seq << 16) | partition, then the item count): every non-empty partition
    of every sequence exactly once (one item for an empty context), in
    non-increasing order of its length in blocks."""
    lens = [0, 5, 600, 1500, 40, 2100, 16, 17]
    w = W.decode_workload("plan", lens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                          dtype="bf16", seed=61)
    d = DeviceStep(w).step()
    S, P, Hq, D = len(lens), 512, 8, 128
    max_ctx = w.max_context_len
    ws = pa.alloc_workspace(S, Hq, D, max_ctx, P, "cuda", persistent=True)
    ws.fill_(0xFF)
    _persistent(d, ws=ws)
    parts = -(-max_ctx // P)
    base = pa.decode_workspace_size(S, Hq, D, max_ctx, P)
    items_bytes = S * parts * 4
    host = ws.cpu().numpy()
    items = host[base:base + items_bytes].view(np.int32)
    plan = host[base + (-(-items_bytes // 256)) * 256:][:8].view(np.int32)
    pb = P // 16
    want = {}
    for s, L in enumerate(lens):
        nblk = -(-L // 16)
        n = max(1, -(-nblk // pb))
        for p in range(n):
            want[(s, p)] = min(pb, nblk - p * pb) if nblk else 0
    assert int(plan[0]) == len(want)
    got = [(int(v) >> 16, int(v) & 0xFFFF) for v in items[:len(want)]]
    assert sorted(got) == sorted(want)
    sizes = [want[i] for i in got]
    assert all(a >= b for a, b in zip(sizes, sizes[1:])), sizes
