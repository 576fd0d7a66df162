"""Seeded synthetic inputs for the paged decode step.

This module only builds inputs: block tables from a toy allocator, context
lengths, the paged K/V pool as it stands before the step, the new tokens'
K/V rows with the cache slots they go to, the queries and the copy-on-write
pairs. It computes no attention and shares nothing with either the CUDA
library or the CPU oracle, both of which consume what it returns.

Every tensor of 16-bit values is returned as ``uint16`` bit patterns so the
GPU and the oracle see identical bits. Values are N(0, 1) rounded once
(round-to-nearest-even) to fp16 or bf16.

Cache layout (block-major): ``pool[physical_block, kv_head, slot, d]`` with
16 slots per block ("Optimizing LLM Inference: From PagedAttention to AI
Infra", "On-Demand Allocation": 16-token blocks). A token at logical
position ``t`` of a sequence lives in slot ``t % 16`` of physical block
``block_table[t // 16]`` (same page, Figure 2), and its flat slot number is
``physical_block * 16 + t % 16``.

Slots that hold no token of any sequence (the unused tail of each last
block, blocks no table references, and the slots this step will write) are
filled with a NaN pattern, so that a kernel which reads a slot it must not
use produces NaN instead of a plausible number.

Step semantics (one decode step of one layer):
  1. ``copy_blocks(copy_pairs)``   -- copy-on-write forks, if any;
  2. ``write_kv(new_k, new_v, slot_mapping)`` -- store this step's tokens;
  3. ``decode(q, block_tables, context_lens)`` -- ``context_lens`` already
     counts the tokens written in step 2.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BLOCK_SIZE = 16
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


@dataclass
class DecodeWorkload:
    name: str
    dtype: str                  # "f16" or "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    partition_tokens: int
    scale: float
    context_lens: np.ndarray    # int32 [S], after this step's writes
    block_tables: np.ndarray    # int32 [S, stride], unused entries = -1
    k_pool: np.ndarray          # uint16 [NB, H_kv, 16, D], before the step
    v_pool: np.ndarray
    q: np.ndarray               # uint16 [S, H_q, D]
    new_k: np.ndarray           # uint16 [T, H_kv, D]
    new_v: np.ndarray
    slot_mapping: np.ndarray    # int64 [T]
    copy_pairs: np.ndarray      # int64 [n, 2] (src, dst)
    seed: int = 0
    notes: dict = field(default_factory=dict)
    block_size: int = BLOCK_SIZE
    q_start: np.ndarray | None = None  # int32 [S+1] for query chunks; None = one token each

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def elem_bytes(self) -> int:
        return 2

    def kv_bytes(self) -> int:
        """K and V bytes one decode step must read: every valid token, every
        KV head, K and V, D elements of 2 bytes."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * 2 * \
            self.head_dim * self.elem_bytes

    def unique_kv_bytes(self) -> int:
        """K and V bytes of the distinct cache slots the decode reads (blocks
        shared by several tables counted once)."""
        used = {}
        for s, L in enumerate(self.context_lens):
            L = int(L)
            for j in range(-(-L // self.block_size)):
                p = int(self.block_tables[s, j])
                used[p] = max(used.get(p, 0), min(self.block_size, L - j * self.block_size))
        return sum(used.values()) * self.num_kv_heads * 2 * self.head_dim * self.elem_bytes

    def step_bytes(self) -> dict:
        """Algorithmic bytes per step, by operation."""
        S, Hq, D, Hkv = self.num_seqs, self.num_q_heads, self.head_dim, self.num_kv_heads
        T = int(self.slot_mapping.shape[0])
        n_pairs = int(self.copy_pairs.shape[0])
        blk = Hkv * self.block_size * D * self.elem_bytes
        Tq = int(self.q.shape[0])  # query rows: S for decode, sum of chunk lengths otherwise
        return {
            "decode": self.kv_bytes() + 2 * Tq * Hq * D * self.elem_bytes
            + S * 4 + int((np.ceil(self.context_lens / self.block_size)).sum()) * 4,
            "write_kv": 2 * 2 * T * Hkv * D * self.elem_bytes + T * 8,
            "copy_blocks": 2 * 2 * n_pairs * blk + n_pairs * 16,
        }


def _round_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 -> fp16 / bf16 bit patterns, round-to-nearest-even (library casts)."""
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _normal_bits(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 26
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = _round_bits(rng.standard_normal(m, dtype=np.float32), dtype)
    return out.reshape(shape)


def blocks_needed(num_tokens: int, block_size: int = BLOCK_SIZE) -> int:
    """Blocks a context of ``num_tokens`` tokens occupies when blocks are
    handed out only as the previous one fills ("On-Demand Allocation")."""
    return -(-int(num_tokens) // block_size)


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, num_tokens: int,
                   dtype_bytes: int) -> int:
    """KV-cache size of one sequence: 2 (K and V) x layers x KV heads x head
    dim x tokens x bytes per value ("Understanding KV Cache ...", and "The
    KV Cache: The Trillion-Dollar Bottleneck")."""
    return 2 * num_layers * num_kv_heads * head_dim * num_tokens * dtype_bytes


class ToyBlockAllocator:
    """A pool of same-sized physical blocks handed out in a seeded random
    order, so that logically adjacent blocks are physically scattered
    ("Fixed Block Size, Mitigating External Fragmentation": freed blocks go
    back to a pool of identical blocks). Only used to build inputs."""

    def __init__(self, num_blocks: int, rng: np.random.Generator):
        self.num_blocks = int(num_blocks)
        self._free = list(rng.permutation(self.num_blocks).astype(np.int64))

    def allocate(self, n: int) -> np.ndarray:
        if n > len(self._free):
            raise MemoryError(f"toy pool exhausted: want {n}, have {len(self._free)}")
        out, self._free = self._free[:n], self._free[n:]
        return np.asarray(out, dtype=np.int64)

    def free(self, ids) -> None:
        self._free.extend(int(i) for i in ids)

    @property
    def num_free(self) -> int:
        return len(self._free)


def slot_of(block_table_row: np.ndarray, position: int, block_size: int = BLOCK_SIZE) -> int:
    """Flat cache slot of logical token ``position`` of one sequence."""
    return int(block_table_row[position // block_size]) * block_size + position % block_size


def _fills_for(tables, valid_lens):
    """(physical block, slots already holding tokens) for every block the
    tables reach within each sequence's valid prefix; a block shared by
    several tables is listed once."""
    seen, fills = set(), []
    for t, n_valid in zip(tables, valid_lens):
        n_valid = int(n_valid)
        for j in range(blocks_needed(n_valid)):
            p = int(t[j])
            if p not in seen:
                seen.add(p)
                fills.append((p, min(BLOCK_SIZE, n_valid - j * BLOCK_SIZE)))
    return fills


def _build(name, dtype, Hq, Hkv, D, partition_tokens, seed, rng, tables, fills,
           context_lens, num_blocks, writes, copy_pairs, notes) -> DecodeWorkload:
    """Assemble a workload.

    ``tables``: list of int64 arrays (physical ids per logical block);
    ``fills``: (physical block, n) pairs -- the first ``n`` slots of that
    block hold tokens before the step and get random values; every other
    slot of the pool is NaN-filled;
    ``writes``: list of (seq, position) this step writes, in token order."""
    S = len(tables)
    stride = max(1, max(len(t) for t in tables))
    bt = np.full((S, stride), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    nan = NAN_BITS[dtype]
    k_pool = np.full((num_blocks, Hkv, BLOCK_SIZE, D), nan, dtype=np.uint16)
    v_pool = np.full_like(k_pool, nan)
    full = np.array([p for p, n in fills if n == BLOCK_SIZE], dtype=np.int64)
    if full.size:
        k_pool[full] = _normal_bits(rng, (full.size, Hkv, BLOCK_SIZE, D), dtype)
        v_pool[full] = _normal_bits(rng, (full.size, Hkv, BLOCK_SIZE, D), dtype)
    for p, n in fills:
        if 0 < n < BLOCK_SIZE:
            k_pool[p, :, :n, :] = _normal_bits(rng, (Hkv, n, D), dtype)
            v_pool[p, :, :n, :] = _normal_bits(rng, (Hkv, n, D), dtype)
    T = len(writes)
    slot_mapping = np.array([slot_of(bt[s], pos) for s, pos in writes], dtype=np.int64)
    new_k = _normal_bits(rng, (T, Hkv, D), dtype)
    new_v = _normal_bits(rng, (T, Hkv, D), dtype)
    q = _normal_bits(rng, (S, Hq, D), dtype)
    cp = np.asarray(copy_pairs, dtype=np.int64).reshape(-1, 2)
    return DecodeWorkload(name=name, dtype=dtype, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          partition_tokens=partition_tokens, scale=1.0 / float(np.sqrt(D)),
                          context_lens=np.asarray(context_lens, dtype=np.int32), block_tables=bt,
                          k_pool=k_pool, v_pool=v_pool, q=q, new_k=new_k, new_v=new_v,
                          slot_mapping=slot_mapping.reshape(-1), copy_pairs=cp, seed=seed,
                          notes=notes)


def decode_workload(name: str, context_lens, *, num_q_heads: int, num_kv_heads: int,
                    head_dim: int, dtype: str, seed: int, pool_factor: float = 1.5,
                    num_blocks: int | None = None, partition_tokens: int = 512,
                    rng: np.random.Generator | None = None) -> DecodeWorkload:
    """Independent sequences, each writing one new token this step: the
    context before the step is ``context_lens - 1`` tokens, the new token
    goes to position ``context_lens - 1``."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int64)
    need = [blocks_needed(int(L)) for L in lens]
    nb = num_blocks if num_blocks is not None else max(1, int(np.ceil(pool_factor * sum(need))))
    alloc = ToyBlockAllocator(nb, rng)
    tables = [alloc.allocate(n) for n in need]
    writes = [(s, int(L) - 1) for s, L in enumerate(lens) if L > 0]
    return _build(name, dtype, num_q_heads, num_kv_heads, head_dim, partition_tokens, seed, rng,
                  tables, _fills_for(tables, np.maximum(lens - 1, 0)), lens, nb, writes, [],
                  {"pool_factor": pool_factor, "blocks_used": int(sum(need))})


def chunk_workload(name: str, context_lens, query_lens, *, num_q_heads: int, num_kv_heads: int,
                   head_dim: int, dtype: str, seed: int, pool_factor: float = 1.5,
                   partition_tokens: int = 512,
                   rng: np.random.Generator | None = None) -> DecodeWorkload:
    """Each sequence's last ``query_lens[s]`` context tokens are written this
    step and are the queries (a prompt chunk, or draft tokens to verify);
    ``context_lens`` counts them. q has sum(query_lens) rows, sequence s owning
    rows ``q_start[s]:q_start[s+1]``."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int64)
    tq = np.asarray(query_lens, dtype=np.int64)
    assert (tq >= 0).all() and (tq <= lens).all()
    need = [blocks_needed(int(L)) for L in lens]
    nb = max(1, int(np.ceil(pool_factor * sum(need))))
    alloc = ToyBlockAllocator(nb, rng)
    tables = [alloc.allocate(n) for n in need]
    writes = [(s, int(p)) for s in range(len(lens)) for p in range(int(lens[s] - tq[s]), int(lens[s]))]
    w = _build(name, dtype, num_q_heads, num_kv_heads, head_dim, partition_tokens, seed, rng,
               tables, _fills_for(tables, lens - tq), lens, nb, writes, [],
               {"pool_factor": pool_factor, "query_lens": tq.tolist()})
    w.q = _normal_bits(rng, (int(tq.sum()), num_q_heads, head_dim), dtype)
    w.q_start = np.concatenate([[0], np.cumsum(tq)]).astype(np.int32)
    return w


def spec_verify(seed: int = 396, batch: int = 256, draft: int = 4) -> DecodeWorkload:
    """Speculative-decoding verification on the Llama-3-8B-shaped GQA batch:
    each of 256 sequences (lognormal lengths, median 1024) checks ``draft``
    proposed tokens in one pass; with 4 query heads per KV head, 4 tokens fill
    one 16-row tile. Split-K partitions of 2048 tokens: a partition's merge of
    16 rows costs four times a decode tile's, so longer partitions pay it
    less often (the 256 x 8 (sequence, KV head) pairs still fill the GPU)."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.round(np.exp(np.log(1024.0) + rng.standard_normal(batch))),
                   16, 8192).astype(np.int64)
    return chunk_workload("spec_verify", lens, np.full(batch, draft), num_q_heads=32,
                          num_kv_heads=8, head_dim=128, dtype="bf16", seed=seed, rng=rng,
                          partition_tokens=2048)


def chunked_prefill(seed: int = 397, batch: int = 16, chunk: int = 256) -> DecodeWorkload:
    """Chunked prefill on the Llama-3-8B shape: 16 prompts of 1024..8192
    tokens, each processing its next ``chunk`` prompt tokens against the
    prefix already cached."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1024, 8192, size=batch, endpoint=True)
    # 16 sequences x 8 KV heads x 8 query tiles already fill the GPU: no split-K
    return chunk_workload("chunked_prefill", lens, np.full(batch, chunk), num_q_heads=32,
                          num_kv_heads=8, head_dim=128, dtype="bf16", seed=seed, rng=rng,
                          partition_tokens=0)


# ---------------------------------------------------------------------------
# The five named configurations.
# ---------------------------------------------------------------------------

def tiny(seed: int = 391) -> DecodeWorkload:
    """4 sequences with {7, 16, 33, 50} cached tokens, H_q = H_kv = 4, D = 64,
    fp16, a 32-block pool handed out in a seeded random order. Each sequence
    writes one new token (so decode runs over {8, 17, 34, 51}); sequence 1
    crosses into a fresh block. A fifth sequence is a fork of sequence 3
    taken at 50 tokens: it shares sequence 3's three full blocks, and its
    partially filled fourth block is copied to a fresh block before the two
    sequences write different new tokens at position 50."""
    rng = np.random.default_rng(seed)
    before = [7, 16, 33, 50]
    alloc = ToyBlockAllocator(32, rng)
    tables = [alloc.allocate(blocks_needed(L + 1)) for L in before]
    fork_block = alloc.allocate(1)
    tables.append(np.concatenate([tables[3][:3], fork_block]))
    # the fork's private block gets its first two tokens from the copy
    fills = _fills_for(tables[:4], before)
    lens = [L + 1 for L in before] + [51]
    writes = [(s, before[s]) for s in range(4)] + [(4, 50)]
    pairs = [[int(tables[3][3]), int(fork_block[0])]]
    return _build("tiny", "f16", 4, 4, 64, 512, seed, rng, tables, fills, lens, 32, writes, pairs,
                  {"fork_of": 3, "fork_at": 50})


def mha(seed: int = 392, batch: int = 64) -> DecodeWorkload:
    """Llama-2-7B-shaped multi-head decode, one layer: batch 64, 32 heads,
    D = 128, fp16, context lengths uniform in [128, 2048], blocks drawn at
    random from a pool 1.5x the number needed."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048, size=batch, endpoint=True)
    return decode_workload("mha", lens, num_q_heads=32, num_kv_heads=32, head_dim=128,
                           dtype="f16", seed=seed, pool_factor=1.5, rng=rng)


def gqa(seed: int = 393, batch: int = 256, sigma: float = 1.0) -> DecodeWorkload:
    """Llama-3-8B-shaped grouped-query decode, one layer: batch 256, 32 query
    heads over 8 KV heads, D = 128, bf16, context lengths lognormal with
    median 1024 (sigma 1.0 in natural log) clipped to [16, 8192]."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.round(np.exp(np.log(1024.0) + sigma * rng.standard_normal(batch))),
                   16, 8192).astype(np.int64)
    return decode_workload("gqa", lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                           dtype="bf16", seed=seed, pool_factor=1.5, rng=rng)


def shared_prefix(seed: int = 394, num_seqs: int = 100, prefix: int = 5000,
                  suffix_lo: int = 16, suffix_hi: int = 512, num_q_heads: int = 32,
                  num_kv_heads: int = 8, head_dim: int = 128,
                  dtype: str = "bf16") -> DecodeWorkload:
    """100 sequences whose tables share one 5000-token prefix (313 blocks, the
    last one holding 8 tokens) plus unique suffixes uniform in [16, 512]
    tokens; H_q = 32, H_kv = 8, D = 128, bf16 ("KV Cache Sharing
    (Copy-on-Write)": 100 users on one 5,000-token system prompt).

    The cache is taken as it stands at a decode step of these sequences: each
    sequence was forked from the prefix by a copy of the partial prefix block
    into a block of its own (``notes["fork_pairs"]``, one (src, dst) pair per
    sequence, as ``copy_blocks`` makes it: the copy's first 8 slots are the
    shared block's bits), and every suffix token but the last is already
    cached, the copy's free slots first. The step writes each sequence's
    newest token and decodes; the 312 full prefix blocks stay shared and
    unchanged. The fork itself happened before this step, so the step has no
    copy pairs. (Other head counts, head sizes and dtypes for tests.)"""
    rng = np.random.default_rng(seed)
    suf = rng.integers(suffix_lo, suffix_hi, size=num_seqs, endpoint=True)
    n_prefix_blocks = blocks_needed(prefix)
    full = prefix // BLOCK_SIZE
    tail = prefix % BLOCK_SIZE
    lens = prefix + suf
    need_private = [blocks_needed(int(L)) - full for L in lens]
    nb = int(np.ceil(1.5 * (n_prefix_blocks + sum(need_private))))
    alloc = ToyBlockAllocator(nb, rng)
    shared = alloc.allocate(n_prefix_blocks)
    tables, forks = [], []
    for s in range(num_seqs):
        private = alloc.allocate(need_private[s])
        tables.append(np.concatenate([shared[:full], private]))
        if tail:
            forks.append([int(shared[full]), int(private[0])])
    writes = [(s, int(L) - 1) for s, L in enumerate(lens)]
    # Before the step: the shared prefix, and each sequence's own blocks up to
    # its newest token (exclusive). A private copy of the partial prefix
    # block is filled like any block here; its first `tail` slots are then
    # overwritten with the shared block's bits, as the fork's copy left them.
    fills = _fills_for([t[full:] for t in tables], np.maximum(lens - 1 - full * BLOCK_SIZE, 0))
    fills += [(int(p), BLOCK_SIZE) for p in shared[:full]]
    if tail:
        fills.append((int(shared[full]), tail))
    w = _build("shared_prefix", dtype, num_q_heads, num_kv_heads, head_dim, 512, seed, rng,
               tables, fills, lens, nb, writes, [],
               {"prefix": prefix, "shared_blocks": full,
                "partial_prefix_block": int(shared[full]) if tail else -1,
                "fork_pairs": forks})
    for src, dst in forks:
        w.k_pool[dst, :, :tail] = w.k_pool[src, :, :tail]
        w.v_pool[dst, :, :tail] = w.v_pool[src, :, :tail]
    return w


def long_context(seed: int = 395, batch: int = 8, lo: int = 32768, hi: int = 131072,
                 pool_factor: float = 1.25) -> DecodeWorkload:
    """Long-context 70B-shaped grouped-query decode, one layer: batch 8, 64
    query heads over 8 KV heads, D = 128, bf16, context lengths uniform in
    [32768, 131072], scattered blocks, split into 512-token partitions that a
    log-sum-exp reduce combines; one new token written per sequence."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi, size=batch, endpoint=True)
    return decode_workload("long", lens, num_q_heads=64, num_kv_heads=8, head_dim=128,
                           dtype="bf16", seed=seed, pool_factor=pool_factor, rng=rng)


def skewed(seed: int = 398, batch: int = 256, n_long: int = 4, long_lo: int = 65536,
           long_hi: int = 131072, short_median: float = 512.0, sigma: float = 0.7,
           short_hi: int = 4096) -> DecodeWorkload:
    """A decode batch of mixed lengths on the Llama-3-8B GQA shape (32 query
    heads over 8 KV heads, D = 128, bf16): ``n_long`` long-context requests
    uniform in [65536, 131072] tokens among short ones, lognormal with median
    512 (sigma 0.7) clipped to [16, 4096]; the long ones sit at random batch
    positions. max_context_len is set by the longest, so a grid sized by it
    holds mostly empty partitions: the case a work-queue schedule is for.
    Split-K partitions of 2048 tokens (the long rows then reduce 56
    partitions, not 223)."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.round(np.exp(np.log(short_median) + sigma * rng.standard_normal(batch))),
                   16, short_hi).astype(np.int64)
    where = rng.choice(batch, size=n_long, replace=False)
    lens[where] = rng.integers(long_lo, long_hi, size=n_long, endpoint=True)
    return decode_workload("skewed", lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                           dtype="bf16", seed=seed, pool_factor=1.25, rng=rng,
                           partition_tokens=2048)


CONFIGS = {
    "tiny": tiny,
    "mha": mha,
    "gqa": gqa,
    "shared_prefix": shared_prefix,
    "long": long_context,
    "spec_verify": spec_verify,
    "chunked_prefill": chunked_prefill,
    "skewed": skewed,
}


def make(name: str, **kw) -> DecodeWorkload:
    return CONFIGS[name](**kw)
