"""GPU parity of pa_decode_shared_prefix: decode of a batch whose sequences
all begin with the same blocks (many users of one prompt, their copy-on-write
forks sharing every full prefix block: "PagedAttention" guide, "KV Cache
Sharing (Copy-on-Write)"). The whole partitions inside the shared prefix run
as one tcgen05 contraction over all sequences' queries, the rest as decode
partitions, merged by the reduce: the oracle's decode within the decode
tolerance; pa_decode's bits where the call falls back to it."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, assert_decode_close, oracle_caches_after_step, to_f64

pytestmark = pytest.mark.gpu


def _shared_tokens(w):
    return int(w.notes["shared_blocks"]) * pa.PA_BLOCK_SIZE


def _decode(d, P, shared, bt=None, cl=None):
    w = d.w
    out = torch.full_like(d.out, float("nan"))
    d.err.zero_()
    pa.decode(out, d.q, d.k_cache, d.v_cache, d.bt if bt is None else bt,
              d.cl if cl is None else cl, scale=w.scale, max_context_len=w.max_context_len,
              partition_tokens=P, dev_error=d.err, shared_prefix_tokens=shared)
    torch.cuda.synchronize()
    return out


def _oracle(w):
    kc, vc = oracle_caches_after_step(w)
    return oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)


@pytest.mark.parametrize("P", [256, 512, 1024])
def test_shared_prefix_matches_the_oracle(P):
    """2,096 shared tokens: 8, 4 and 2 shared partitions; 24 sequences x 4
    query heads per KV head = 96 rows of the contraction."""
    w = W.shared_prefix(num_seqs=24, prefix=2100, suffix_hi=300, seed=31 + P)
    d = DeviceStep(w, P)
    d.cache_ops()
    out = _decode(d, P, _shared_tokens(w))
    assert int(d.err.item()) == 0
    assert_decode_close(to_f64(out), _oracle(w), f"shared prefix, P={P}")
    plain = _decode(d, P, 0)
    assert_decode_close(to_f64(out), to_f64(plain), f"against pa_decode, P={P}")


@pytest.mark.parametrize("P,shared", [(2048, None), (512, 1000), (512, 0)])
def test_fewer_than_two_shared_partitions_run_pa_decode(P, shared):
    """A prefix spanning fewer than two whole partitions (or none given): the
    call is pa_decode, bit for bit."""
    w = W.shared_prefix(num_seqs=24, prefix=2100, suffix_hi=300, seed=41)
    d = DeviceStep(w, P)
    d.cache_ops()
    a = _decode(d, P, _shared_tokens(w) if shared is None else shared)
    b = _decode(d, P, 0)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert int(d.err.item()) == 0


@pytest.mark.parametrize("Hq,Hkv,dtype,S", [(8, 8, "f16", 64), (32, 4, "bf16", 12),
                                             (32, 2, "f16", 8), (16, 4, "f16", 20)])
def test_shared_prefix_group_sizes_and_fp16(Hq, Hkv, dtype, S):
    w = W.shared_prefix(num_seqs=S, prefix=1800, suffix_hi=260, num_q_heads=Hq,
                        num_kv_heads=Hkv, dtype=dtype, seed=Hq + Hkv + S)
    d = DeviceStep(w, 256)
    d.cache_ops()
    out = _decode(d, 256, _shared_tokens(w))
    assert int(d.err.item()) == 0
    assert_decode_close(to_f64(out), _oracle(w), f"Hq={Hq} Hkv={Hkv} {dtype}")


def test_ineligible_calls_run_pa_decode():
    """D 64, or fewer than 64 rows of (sequence, head) per KV head: pa_decode."""
    for kw in (dict(num_seqs=24, head_dim=64), dict(num_seqs=12, num_q_heads=8, num_kv_heads=2)):
        w = W.shared_prefix(prefix=1500, suffix_hi=200, seed=51, **kw)
        d = DeviceStep(w, 256)
        d.cache_ops()
        a = _decode(d, 256, _shared_tokens(w))
        b = _decode(d, 256, 0)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), kw


def test_a_sequence_off_the_shared_prefix_is_counted_once():
    """Sequence 3's table differs inside the shared partitions, sequence 5's
    context is shorter than them: each is counted once; every other
    sequence's output is still its attention."""
    w = W.shared_prefix(num_seqs=24, prefix=2100, suffix_hi=300, seed=61)
    d = DeviceStep(w, 512)
    d.cache_ops()
    bt = d.bt.clone()
    own_last = (int(w.context_lens[3]) + 15) // 16 - 1
    bt[3, 7] = int(w.block_tables[3, own_last])   # a valid block of sequence 3's own
    cl = d.cl.clone()
    cl[5] = 300
    out = _decode(d, 512, _shared_tokens(w), bt=bt, cl=cl)
    assert int(d.err.item()) == 2
    ref = _oracle(w)
    keep = [s for s in range(w.num_seqs) if s not in (3, 5)]
    assert_decode_close(to_f64(out)[keep], ref[keep], "the other sequences")


def test_full_size_shared_prefix_sampled():
    """The shared-prefix config at full size (100 sequences on one
    5000-token prompt, 512-token partitions: 9 shared), sampled sequences."""
    w = W.shared_prefix()
    d = DeviceStep(w)
    d.cache_ops()
    out = _decode(d, w.partition_tokens, _shared_tokens(w))
    assert int(d.err.item()) == 0
    rng = np.random.default_rng(3)
    seqs = sorted(set(rng.choice(w.num_seqs, size=10, replace=False).tolist())
                  | {0, w.num_seqs - 1})
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q[seqs], kc, vc, w.block_tables[seqs], w.context_lens[seqs], w.scale,
                        w.dtype)
    assert_decode_close(to_f64(out)[seqs], ref, "full-size shared prefix")


def test_a_prefix_that_is_the_whole_context():
    """Every context is exactly the 2,048 shared tokens: of its four 512-token
    partitions the first three are shared and the last is left to the decode
    kernel (it always keeps the longest context's last partition)."""
    w = W.shared_prefix(num_seqs=24, prefix=2100, suffix_hi=300, seed=71)
    d = DeviceStep(w, 512)
    d.cache_ops()
    L = 2048
    cl = torch.full_like(d.cl, L)
    out = torch.full_like(d.out, float("nan"))
    d.err.zero_()
    pa.decode(out, d.q, d.k_cache, d.v_cache, d.bt, cl, scale=w.scale, max_context_len=L,
              partition_tokens=512, dev_error=d.err, shared_prefix_tokens=L)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, np.full(w.num_seqs, L, np.int32), w.scale,
                        w.dtype)
    assert_decode_close(to_f64(out), ref, "prefix = whole context")
