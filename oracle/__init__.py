"""fp64 CPU oracle for the paged-KV-cache decode hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code
with the CUDA library (``paged_kv_cache_391_b200``) and never imports it.

The arithmetic lives in ``pa_oracle.c`` (plain C, double precision, compiled
with gcc into ``liboracle.so``); this module only marshals numpy arrays.
What each function follows, by page and section:

* ``write_kv`` -- "Optimizing LLM Inference: From PagedAttention to AI Infra",
  "Understanding KV Cache ...": each decode step stores the new token's K and
  V at every layer, so later steps read them instead of recomputing them.
* ``copy_blocks`` -- same page, "Copy-on-Write"; and "PagedAttention"
  (ai-system-design-guide), "KV Cache Sharing (Copy-on-Write)": a shared block
  is copied when one sequence diverges, the shared original stays unchanged.
* ``swap_blocks`` -- "PagedAttention", "Managing Virtual Memory (Block
  Manager)": blocks move between GPU memory and CPU RAM and back.
* ``prefill_chunk`` -- "PagedAttention in Action ...", "Chunked Prefill", and
  "The Memory Wall ...", "The Next Frontier: Speculative Decoding and Beyond":
  the last Tq tokens of a context are queries at once, each seeing the context
  up to its own position.
* ``decode`` -- same first page, "PagedAttention: Decoupling Logical Context
  from Contiguous GPU Memory" (Figure 2), and "The Memory Wall ...", "How it
  Works Under the Hood" and "Show Me The Code": the kernel walks the block
  table in logical order, so the result is ordinary attention over the
  logically contiguous context.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16 = 0
BF16 = 1
DTYPES = {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}


def build(force: bool = False) -> str:
    """Compile ``pa_oracle.c`` into ``liboracle.so`` (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-pthread",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64 = ctypes.c_int32, ctypes.c_int64
            lib.oracle_decode16.argtypes = [P, i64, ctypes.c_int, P]
            lib.oracle_decode16.restype = None
            lib.oracle_write_kv.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64]
            lib.oracle_write_kv.restype = i64
            lib.oracle_copy_blocks.argtypes = [P, P, i32, P, i32, i32, i32, i32]
            lib.oracle_copy_blocks.restype = None
            lib.oracle_swap_blocks.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32]
            lib.oracle_swap_blocks.restype = None
            lib.oracle_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                          ctypes.c_double, ctypes.c_int, P, i64, ctypes.c_int]
            lib.oracle_decode.restype = ctypes.c_int
            lib.oracle_num_cores.argtypes = []
            lib.oracle_num_cores.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    return DTYPES[str(dtype)]


def num_cores() -> int:
    return int(_load().oracle_num_cores())


def decode16(bits: np.ndarray, dtype) -> np.ndarray:
    """Exact decode of fp16 / bf16 bit patterns (uint16) to float64."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_decode16(_ptr(bits), bits.size, _dtype_code(dtype), _ptr(out))
    return out


def write_kv(k, v, k_cache, v_cache, slot_mapping, block_size: int = 16) -> int:
    """Scatter new K/V rows ``[T, H_kv, D]`` (uint16 bits) into the caches
    ``[NB, H_kv, block_size, D]`` in place. Returns the count of out-of-range
    slots (negative slots are padding and are skipped silently)."""
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    T, H, D = k.shape
    NB = k_cache.shape[0]
    return int(_load().oracle_write_kv(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(slot_mapping), T, H, D, block_size, NB))


def copy_blocks(k_caches, v_caches, block_mapping, block_size: int = 16) -> None:
    """Copy whole physical blocks ``src -> dst`` for every ``(src, dst)`` row of
    ``block_mapping`` in every layer's K and V cache (lists of arrays), in place."""
    block_mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    L = len(k_caches)
    kp = (ctypes.c_void_p * L)(*[_ptr(c) for c in k_caches])
    vp = (ctypes.c_void_p * L)(*[_ptr(c) for c in v_caches])
    _, H, bs, D = k_caches[0].shape
    _load().oracle_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                               L, _ptr(block_mapping), block_mapping.shape[0], H, D, bs)


def swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, block_size: int = 16) -> None:
    """Copy whole blocks ``src -> dst`` from per-layer source pools into
    per-layer destination pools (lists of ``[NB, H_kv, 16, D]`` uint16 arrays;
    the two sides may have different block counts), in place."""
    block_mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    L = len(src_k)
    arrs = [(ctypes.c_void_p * L)(*[_ptr(c) for c in side]) for side in (src_k, src_v, dst_k, dst_v)]
    _, H, bs, D = src_k[0].shape
    _load().oracle_swap_blocks(*[ctypes.cast(a, ctypes.c_void_p) for a in arrs], L,
                               _ptr(block_mapping), block_mapping.shape[0], H, D, bs)


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype,
           num_kv_heads: int | None = None, rows=None, n_threads: int = 0) -> np.ndarray:
    """Paged decode attention in float64.

    ``q``: uint16 bits ``[S, H_q, D]``; caches ``[NB, H_kv, 16, D]``;
    ``block_tables`` int32 ``[S, stride]``; ``context_lens`` int32 ``[S]``.
    Returns ``[S, H_q, D]`` float64, or ``[len(rows), D]`` when ``rows`` (a list
    of flat ``seq * H_q + head`` indices) is given.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and (num_kv_heads is None or num_kv_heads == Hkv) and Hq % Hkv == 0
    if rows is None:
        out = np.empty((S, Hq, D), dtype=np.float64)
        rows_p, nrows = None, S * Hq
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((rows.size, D), dtype=np.float64)
        rows_p, nrows = _ptr(rows), rows.size
    rc = _load().oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                               _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                               S, Hq, Hkv, D, bs, NB, float(scale), _dtype_code(dtype),
                               rows_p, nrows, int(n_threads))
    if rc != 0:
        raise ValueError("oracle.decode: a block-table entry is outside [0, num_blocks)")
    return out


def prefill_chunk(q, q_start, k_cache, v_cache, block_tables, context_lens, scale: float, dtype,
                  rows=None, n_threads: int = 0) -> np.ndarray:
    """Attention of each sequence's last Tq context tokens, causal in the chunk.

    ``q``: uint16 bits ``[T, H_q, D]`` where sequence s owns rows
    ``q_start[s] .. q_start[s+1]-1``. Query token t of sequence s (t counted
    from the chunk start) attends to context positions
    ``0 .. context_lens[s] - Tq_s + t`` -- i.e. it is the decode of one query
    over the first ``context_lens[s] - Tq_s + t + 1`` tokens of the same
    block table. Returns ``[T, H_q, D]`` float64 (or the requested flat
    ``token * H_q + head`` rows)."""
    q_start = np.asarray(q_start, dtype=np.int64)
    context_lens = np.asarray(context_lens, dtype=np.int64)
    block_tables = np.asarray(block_tables, dtype=np.int32)
    tq = np.diff(q_start)
    tok_seq = np.repeat(np.arange(len(tq)), tq)
    tok_t = np.arange(int(q_start[-1])) - q_start[tok_seq]
    tok_len = (context_lens[tok_seq] - tq[tok_seq] + tok_t + 1).astype(np.int32)
    return decode(q, k_cache, v_cache, block_tables[tok_seq], tok_len, scale, dtype, rows=rows,
                  n_threads=n_threads)
