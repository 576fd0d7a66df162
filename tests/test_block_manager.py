"""The host block manager: the pages' sharing and allocation examples, checked
on both the native manager in libpa and the plain-Python model in oracle/,
then the two compared operation by operation on seeded random workloads.
No GPU needed (host code)."""
import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, OutOfBlocks
from paged_kv_cache_391_b200 import build as pa_build
from paged_kv_cache_391_b200 import pa


class Native:
    """Adapter: the native manager with the model's method names."""

    def __init__(self, n):
        pa_build.build()
        self.m = pa.BlockManager(n)

    def add_sequence(self, sid, n):
        self.m.add_sequence(sid, n)

    def fork(self, p, c):
        self.m.fork(p, c)

    def free(self, sid):
        self.m.free(sid)

    def slot(self, sid, pos):
        return int(self.m.slots(sid, pos, 1)[0])

    def append_slots(self, ids):
        s, c = self.m.append_slots(ids)
        return s.tolist(), [tuple(x) for x in c.tolist()]

    def block_tables(self, ids, stride):
        bt, lens = self.m.block_tables(ids, stride)
        return bt.tolist(), lens.tolist()

    def stats(self):
        return self.m.stats()

    def ref(self, b):
        return self.m.refcount(b)


def make(kind, n):
    if kind == "native":
        return Native(n)
    return BlockManagerModel(n)


def refcount(m, b):
    return m.ref(b) if isinstance(m, Native) else m.ref[b]


def is_out_of_blocks(exc):
    return isinstance(exc, OutOfBlocks) or (isinstance(exc, pa.PaError)
                                            and exc.status == pa.PA_ERR_OUT_OF_BLOCKS)


KINDS = ["native", "model"]


@pytest.mark.parametrize("kind", KINDS)
def test_on_demand_allocation_35_tokens(kind):
    """"On-Demand Allocation": 35 tokens take 3 blocks, 13 slots of the third
    stay free; 13 more tokens need no new block, the 14th does."""
    m = make(kind, 10)
    m.add_sequence(1, 35)
    assert m.stats()["used_blocks"] == 3
    for _ in range(13):
        m.append_slots([1])
    assert m.stats()["used_blocks"] == 3
    m.append_slots([1])
    assert m.stats()["used_blocks"] == 4 and m.stats()["tokens"] == 49


@pytest.mark.parametrize("kind", KINDS)
def test_four_candidates_share_a_1000_token_prompt(kind):
    """"Copy-on-Write": four candidates of one 1000-token prompt reference the
    same blocks; when each writes its first own token, the shared partial
    last block is copied for all but the last holder."""
    m = make(kind, 200)
    m.add_sequence(0, 1000)
    for c in (1, 2, 3):
        m.fork(0, c)
    st = m.stats()
    assert st["used_blocks"] == 63 and st["logical_blocks"] == 4 * 63 and st["shared_blocks"] == 63
    slots, cow = m.append_slots([0, 1, 2, 3])
    assert len(cow) == 3
    last = cow[0][0]
    assert all(src == last for src, _ in cow)
    assert m.stats()["used_blocks"] == 66
    assert len(set(s // 16 for s in slots)) == 4             # four different blocks now
    assert all(s % 16 == 1000 % 16 for s in slots)
    bt, lens = m.block_tables([0, 1, 2, 3], 63)
    assert lens == [1001] * 4
    for j in range(62):                                       # the full blocks stay shared
        assert len({row[j] for row in bt}) == 1 and refcount(m, bt[0][j]) == 4


@pytest.mark.parametrize("kind", KINDS)
def test_100_users_on_a_5000_token_system_prompt(kind):
    """"KV Cache Sharing (Copy-on-Write)": 100 users on one 5,000-token prompt
    store it once (313 blocks, not the 500k tokens of private copies); each
    user's first own token copies only the partially filled last block."""
    m = make(kind, 2000)
    m.add_sequence(0, 5000)
    for u in range(1, 100):
        m.fork(0, u)
    st = m.stats()
    assert st["used_blocks"] == 313 and st["tokens"] == 100 * 5000 == 500000
    _, cow = m.append_slots(list(range(100)))
    assert len(cow) == 99 and m.stats()["used_blocks"] == 313 + 99
    assert m.stats()["shared_blocks"] == 312


@pytest.mark.parametrize("kind", KINDS)
def test_free_returns_everything_and_reuses_last_freed_first(kind):
    m = make(kind, 8)
    m.add_sequence(1, 40)            # blocks 0, 1, 2
    m.fork(1, 2)
    m.free(1)
    assert m.stats()["free_blocks"] == 5
    m.free(2)
    assert m.stats()["free_blocks"] == 8 and m.stats()["sequences"] == 0
    m.add_sequence(3, 1)
    bt, _ = m.block_tables([3], 1)
    assert bt[0][0] == 2             # the last block freed is handed out first


@pytest.mark.parametrize("kind", KINDS)
def test_out_of_blocks_changes_nothing(kind):
    m = make(kind, 5)
    m.add_sequence(1, 48)            # 3 blocks, all full
    m.add_sequence(2, 30)            # 2 blocks
    before = (m.stats(), m.block_tables([1, 2], 5))
    with pytest.raises(Exception) as e:
        m.append_slots([1, 2])       # seq 1 needs a new block, none left
    assert is_out_of_blocks(e.value)
    assert (m.stats(), m.block_tables([1, 2], 5)) == before
    with pytest.raises(Exception) as e:
        m.add_sequence(3, 17)
    assert is_out_of_blocks(e.value)
    assert m.stats() == before[0]


@pytest.mark.parametrize("kind", KINDS)
def test_slots_follow_the_table(kind):
    m = make(kind, 16)
    m.add_sequence(7, 35)
    bt, lens = m.block_tables([7], 4)
    assert lens == [35] and bt[0][3] == -1
    for pos in range(35):
        assert m.slot(7, pos) == bt[0][pos // 16] * 16 + pos % 16


def _random_ops(seed, n_ops=600, pool=300):
    rng = np.random.default_rng(seed)
    ops, live, next_id = [], [], 0
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.15 or not live:
            ops.append(("add", next_id, int(rng.integers(0, 80))))
            live.append(next_id)
            next_id += 1
        elif r < 0.3:
            p = int(rng.choice(live))
            ops.append(("fork", p, next_id))
            live.append(next_id)
            next_id += 1
        elif r < 0.4 and len(live) > 1:
            sid = int(rng.choice(live))
            live.remove(sid)
            ops.append(("free", sid))
        else:
            k = int(rng.integers(1, len(live) + 1))
            ops.append(("append", [int(x) for x in rng.choice(live, size=k, replace=False)]))
    return ops, pool


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_native_matches_model_on_random_workloads(seed):
    ops, pool = _random_ops(seed)
    nat, mod = make("native", pool), make("model", pool)
    live = []
    for op in ops:
        outs = []
        for m in (nat, mod):
            try:
                if op[0] == "add":
                    outs.append(("ok", m.add_sequence(op[1], op[2])))
                elif op[0] == "fork":
                    outs.append(("ok", m.fork(op[1], op[2])))
                elif op[0] == "free":
                    outs.append(("ok", m.free(op[1])))
                else:
                    outs.append(("ok", m.append_slots(op[1])))
            except Exception as e:                           # noqa: BLE001
                outs.append(("oob" if is_out_of_blocks(e) else "err", None))
        assert outs[0] == outs[1], op
        if outs[0][0] == "ok":
            if op[0] in ("add", "fork"):
                live.append(op[-1] if op[0] == "fork" else op[1])
            elif op[0] == "free":
                live.remove(op[1])
        assert nat.stats() == mod.stats()
        if live:
            assert nat.block_tables(live, 64) == mod.block_tables(live, 64)
    for b in range(pool):
        assert nat.ref(b) == mod.ref[b]
