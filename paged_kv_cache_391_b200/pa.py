"""Thin ctypes binding of libpa (include/pa.h): argument marshalling only.

Every step of the hot path runs in libpa's CUDA kernels. PyTorch supplies
device memory and the current stream. If libpa.so is missing, every call
raises -- there is no CPU or eager fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

(PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE_TOO_SMALL, PA_ERR_CUDA,
 PA_ERR_OUT_OF_BLOCKS) = range(6)
PA_DTYPE_F16, PA_DTYPE_BF16 = 0, 1
PA_BLOCK_SIZE = 16
PA_MAX_LAYERS = 256
PA_DEV_ERR_TIMEOUT = 1 << 24

# Every entry point include/pa.h declares.
EXPORTS = ("pa_write_kv", "pa_decode_workspace_size", "pa_decode", "pa_copy_blocks",
           "pa_status_string", "pa_last_cuda_error", "pa_decode_static", "pa_swap_blocks",
           "pa_bm_create", "pa_bm_destroy", "pa_bm_num_free_blocks", "pa_bm_add_sequence",
           "pa_bm_fork", "pa_bm_free_sequence", "pa_bm_slots", "pa_bm_append_slots",
           "pa_bm_block_tables", "pa_bm_get_stats", "pa_bm_refcount", "pa_prefill_chunk",
           "pa_decode_persistent_workspace_size", "pa_decode_persistent", "pa_read_probe",
           "pa_prefill_chunk_workspace_size", "pa_decode_shared_prefix")
PA_STATIC_WORKSPACE_BYTES = 32 << 20

_lock = threading.Lock()
_lib = None


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {status_string(status)}"
        if status == PA_ERR_CUDA:
            msg += f" ({last_cuda_error()})"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """Open libpa.so (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_391_b200.build` "
                    "(or __graft_entry__.build()); there is no fallback path")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
            L.pa_write_kv.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64, ctypes.c_int, P, P]
            L.pa_write_kv.restype = ctypes.c_int
            L.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
            L.pa_decode_workspace_size.restype = sz
            L.pa_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, i32,
                                    ctypes.c_float, i32, P, sz, P, ctypes.c_int, P]
            L.pa_decode.restype = ctypes.c_int
            L.pa_decode_persistent_workspace_size.argtypes = [i32, i32, i32, i32, i32]
            L.pa_decode_persistent_workspace_size.restype = sz
            L.pa_decode_persistent.argtypes = L.pa_decode.argtypes
            L.pa_decode_persistent.restype = ctypes.c_int
            L.pa_decode_shared_prefix.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32,
                                                  i64, i32, ctypes.c_float, i32, i32, P, sz, P,
                                                  ctypes.c_int, P]
            L.pa_decode_shared_prefix.restype = ctypes.c_int
            L.pa_prefill_chunk.argtypes = [P, P, P, i32, i32, P, P, P, i32, P, i32, i32, i32,
                                           i32, i32, i64, i32, ctypes.c_float, i32, P, sz, P,
                                           ctypes.c_int, P]
            L.pa_prefill_chunk.restype = ctypes.c_int
            L.pa_prefill_chunk_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32]
            L.pa_prefill_chunk_workspace_size.restype = sz
            L.pa_decode_static.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                           i32, ctypes.c_float, i32, P, ctypes.c_int, P]
            L.pa_decode_static.restype = ctypes.c_int
            L.pa_read_probe.argtypes = [P, sz, i32, P, P, P]
            L.pa_read_probe.restype = ctypes.c_int
            L.pa_copy_blocks.argtypes = [P, P, i32, P, i32, i32, i32, i32, i64, ctypes.c_int, P, P]
            L.pa_copy_blocks.restype = ctypes.c_int
            L.pa_swap_blocks.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i64, i64,
                                         ctypes.c_int, P, P]
            L.pa_swap_blocks.restype = ctypes.c_int
            L.pa_bm_create.argtypes = [i64, i32]
            L.pa_bm_create.restype = P
            L.pa_bm_destroy.argtypes = [P]
            L.pa_bm_destroy.restype = None
            L.pa_bm_num_free_blocks.argtypes = [P]
            L.pa_bm_num_free_blocks.restype = i64
            L.pa_bm_add_sequence.argtypes = [P, i64, i64]
            L.pa_bm_fork.argtypes = [P, i64, i64]
            L.pa_bm_free_sequence.argtypes = [P, i64]
            L.pa_bm_slots.argtypes = [P, i64, i64, i64, P]
            L.pa_bm_append_slots.argtypes = [P, P, i32, P, P, P]
            L.pa_bm_block_tables.argtypes = [P, P, i32, P, i32, P]
            L.pa_bm_get_stats.argtypes = [P, P]
            for f in ("pa_bm_add_sequence", "pa_bm_fork", "pa_bm_free_sequence", "pa_bm_slots",
                      "pa_bm_append_slots", "pa_bm_block_tables", "pa_bm_get_stats"):
                getattr(L, f).restype = ctypes.c_int
            L.pa_bm_refcount.argtypes = [P, i32]
            L.pa_bm_refcount.restype = i32
            L.pa_status_string.argtypes = [ctypes.c_int]
            L.pa_status_string.restype = ctypes.c_char_p
            L.pa_last_cuda_error.argtypes = []
            L.pa_last_cuda_error.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def last_cuda_error() -> str:
    return lib().pa_last_cuda_error().decode()


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_DTYPE_F16
    if t.dtype == torch.bfloat16:
        return PA_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp16 or bf16 only")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpa must be contiguous")
    return t.data_ptr()


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def write_kv(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             slot_mapping: torch.Tensor, *, dev_error: torch.Tensor | None = None,
             stream=None) -> None:
    """Store new rows k, v ``[T, H_kv, D]`` in the caches ``[NB, H_kv, 16, D]`` at
    ``slot_mapping`` (int64 ``[T]``)."""
    T, H, D = k.shape
    NB = k_cache.shape[0]
    assert v.shape == k.shape and k_cache.shape == v_cache.shape == (NB, H, PA_BLOCK_SIZE, D)
    assert slot_mapping.dtype == torch.int64 and slot_mapping.numel() == T
    assert k.dtype == v.dtype == k_cache.dtype == v_cache.dtype
    st = lib().pa_write_kv(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                           T, H, D, PA_BLOCK_SIZE, NB, _dtype_code(k), _ptr(dev_error),
                           _stream(stream, k_cache.device))
    _check(st, "pa_write_kv")


def decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                          partition_tokens: int) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                              partition_tokens))


def decode_persistent_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int,
                                     max_context_len: int, partition_tokens: int) -> int:
    return int(lib().pa_decode_persistent_workspace_size(num_seqs, num_q_heads, head_dim,
                                                         max_context_len, partition_tokens))


def alloc_workspace(num_seqs, num_q_heads, head_dim, max_context_len, partition_tokens,
                    device, persistent: bool = False) -> torch.Tensor | None:
    size = decode_persistent_workspace_size if persistent else decode_workspace_size
    n = size(num_seqs, num_q_heads, head_dim, max_context_len, partition_tokens)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def prefill_chunk_workspace_size(num_q_tokens: int, num_seqs: int, num_q_heads: int,
                                 group_size: int, head_dim: int, max_query_len: int,
                                 max_context_len: int, partition_tokens: int) -> int:
    return int(lib().pa_prefill_chunk_workspace_size(num_q_tokens, num_seqs, num_q_heads,
                                                     group_size, head_dim, max_query_len,
                                                     max_context_len, partition_tokens))


def alloc_chunk_workspace(num_q_tokens, num_seqs, num_q_heads, group_size, head_dim,
                          max_query_len, max_context_len, partition_tokens,
                          device) -> torch.Tensor | None:
    """A workspace for pa_prefill_chunk with room for its longest-first plan."""
    n = prefill_chunk_workspace_size(num_q_tokens, num_seqs, num_q_heads, group_size, head_dim,
                                     max_query_len, max_context_len, partition_tokens)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           block_tables: torch.Tensor, context_lens: torch.Tensor, *, scale: float,
           max_context_len: int, partition_tokens: int = 512,
           workspace: torch.Tensor | None = None, dev_error: torch.Tensor | None = None,
           stream=None, persistent: bool = False,
           shared_prefix_tokens: int = 0) -> torch.Tensor:
    """Paged decode attention: ``out [S, H_q, D] = attention(q, paged K/V)``.
    ``persistent=True`` runs pa_decode_persistent (work-queue schedule, the
    same result bit for bit); its workspace comes from
    ``alloc_workspace(..., persistent=True)``. ``shared_prefix_tokens > 0``
    runs pa_decode_shared_prefix: every sequence starts with that many tokens
    in sequence 0's blocks."""
    S, Hq, D = q.shape
    NB, Hkv = k_cache.shape[:2]
    assert out.shape == q.shape and out.dtype == q.dtype == k_cache.dtype == v_cache.dtype
    assert k_cache.shape == v_cache.shape == (NB, Hkv, PA_BLOCK_SIZE, D)
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2
    assert context_lens.dtype == torch.int32 and context_lens.numel() == S
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    if workspace is None:
        workspace = alloc_workspace(S, Hq, D, max_context_len, partition_tokens, q.device,
                                    persistent)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if shared_prefix_tokens:
        if persistent:
            raise ValueError("shared_prefix_tokens and persistent do not combine")
        st = lib().pa_decode_shared_prefix(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), S, Hq, Hq // Hkv, D, PA_BLOCK_SIZE, NB,
            int(max_context_len), float(scale), int(shared_prefix_tokens), int(partition_tokens),
            _ptr(workspace), ws_bytes, _ptr(dev_error), _dtype_code(q), _stream(stream, q.device))
        _check(st, "pa_decode_shared_prefix")
        return out
    fn = lib().pa_decode_persistent if persistent else lib().pa_decode
    st = fn(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), S, Hq, Hq // Hkv, D, PA_BLOCK_SIZE, NB,
            int(max_context_len), float(scale), int(partition_tokens), _ptr(workspace), ws_bytes,
            _ptr(dev_error), _dtype_code(q), _stream(stream, q.device))
    _check(st, "pa_decode_persistent" if persistent else "pa_decode")
    return out


def prefill_chunk(out: torch.Tensor, q: torch.Tensor, q_start: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, *,
                  scale: float, max_query_len: int, max_context_len: int,
                  partition_tokens: int = 512, workspace: torch.Tensor | None = None,
                  dev_error: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Attention of each sequence's last Tq context tokens (rows
    ``q_start[s]:q_start[s+1]`` of ``q [T, H_q, D]``), causal within the chunk:
    chunked prefill or speculative-draft verification over the paged cache."""
    T, Hq, D = q.shape
    NB, Hkv = k_cache.shape[:2]
    S = context_lens.numel()
    assert out.shape == q.shape and out.dtype == q.dtype == k_cache.dtype == v_cache.dtype
    assert k_cache.shape == v_cache.shape == (NB, Hkv, PA_BLOCK_SIZE, D)
    assert q_start.dtype == torch.int32 and q_start.numel() == S + 1
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    if workspace is None:
        workspace = alloc_chunk_workspace(T, S, Hq, Hq // Hkv, D, max_query_len, max_context_len,
                                          partition_tokens, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().pa_prefill_chunk(_ptr(out), _ptr(q), _ptr(q_start), T, int(max_query_len),
                                _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                block_tables.shape[1], _ptr(context_lens), S, Hq, Hq // Hkv, D,
                                PA_BLOCK_SIZE, NB, int(max_context_len), float(scale),
                                int(partition_tokens), _ptr(workspace), ws_bytes,
                                _ptr(dev_error), _dtype_code(q), _stream(stream, q.device))
    _check(st, "pa_prefill_chunk")
    return out


def decode_static(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, *,
                  scale: float, max_context_len: int, partition_tokens: int = 512,
                  dev_error: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """pa_decode without a caller workspace, for callers that may not allocate
    device memory: the split-K scratch is a fixed array inside libpa
    (PA_STATIC_WORKSPACE_BYTES per GPU). Calls on one device must not overlap
    on the GPU; the first call on a device should precede any stream capture."""
    S, Hq, D = q.shape
    NB, Hkv = k_cache.shape[:2]
    assert out.shape == q.shape and out.dtype == q.dtype == k_cache.dtype == v_cache.dtype
    assert k_cache.shape == v_cache.shape == (NB, Hkv, PA_BLOCK_SIZE, D)
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    st = lib().pa_decode_static(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
                                Hq, Hq // Hkv, D, PA_BLOCK_SIZE, NB, int(max_context_len),
                                float(scale), int(partition_tokens), _ptr(dev_error),
                                _dtype_code(q), _stream(stream, q.device))
    _check(st, "pa_decode_static")
    return out


def read_probe(buf: torch.Tensor, sink: torch.Tensor, *, method: int = 0,
               dev_error: torch.Tensor | None = None, stream=None) -> None:
    """Stream every byte of `buf` (device, contiguous) through the SMs once:
    the memory's read ceiling when timed (method 0: vector loads; 1: bulk
    asynchronous copies into shared memory). `sink`: one device int64."""
    assert buf.is_contiguous() and sink.dtype == torch.int64 and sink.numel() >= 1
    st = lib().pa_read_probe(_ptr(buf), buf.numel() * buf.element_size(), int(method),
                             _ptr(sink), _ptr(dev_error), _stream(stream, buf.device))
    _check(st, "pa_read_probe")


def copy_blocks(k_caches, v_caches, block_mapping: torch.Tensor, *,
                dev_error: torch.Tensor | None = None, stream=None) -> None:
    """Copy whole blocks ``src -> dst`` (int64 ``[n, 2]`` on the device) in every
    layer's K and V cache (lists of ``[NB, H_kv, 16, D]`` tensors)."""
    L = len(k_caches)
    assert L == len(v_caches) and L >= 1
    NB, H, bs, D = k_caches[0].shape
    assert block_mapping.dtype == torch.int64
    n = block_mapping.numel() // 2
    kp = (ctypes.c_void_p * L)(*[_ptr(c) for c in k_caches])
    vp = (ctypes.c_void_p * L)(*[_ptr(c) for c in v_caches])
    st = lib().pa_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                              L, _ptr(block_mapping), n, H, D, bs, NB,
                              _dtype_code(k_caches[0]), _ptr(dev_error),
                              _stream(stream, k_caches[0].device))
    _check(st, "pa_copy_blocks")


def swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping: torch.Tensor, *,
                dev_error: torch.Tensor | None = None, stream=None) -> None:
    """Copy whole blocks ``src -> dst`` between two pools, layer by layer
    (lists of ``[NB, H_kv, 16, D]`` tensors). Each pool lives in device memory
    or in pinned host memory (``tensor.pin_memory()``); ``block_mapping`` is
    an int64 ``[n, 2]`` tensor on the device or in pinned host memory."""
    L = len(src_k)
    assert L >= 1 and len(src_v) == len(dst_k) == len(dst_v) == L
    _, H, bs, D = src_k[0].shape
    assert dst_k[0].shape[1:] == src_k[0].shape[1:]
    assert block_mapping.dtype == torch.int64
    n = block_mapping.numel() // 2
    arrs = [(ctypes.c_void_p * L)(*[_ptr(t) for t in side]) for side in (src_k, src_v, dst_k, dst_v)]
    dev = src_k[0].device if src_k[0].is_cuda else dst_k[0].device
    st = lib().pa_swap_blocks(*[ctypes.cast(a, ctypes.c_void_p) for a in arrs], L,
                              _ptr(block_mapping), n, H, D, bs, src_k[0].shape[0],
                              dst_k[0].shape[0], _dtype_code(src_k[0]), _ptr(dev_error),
                              _stream(stream, dev))
    _check(st, "pa_swap_blocks")


class _BmStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("num_blocks", "free_blocks", "used_blocks",
                                              "shared_blocks", "sequences", "tokens",
                                              "logical_blocks")]


class BlockManager:
    """Host block manager of libpa (pa_bm_*): reference-counted 16-token
    blocks, on-demand allocation, copy-on-write on the first divergent write.
    Produces the host arrays the kernels consume (slot mapping, copy pairs,
    block tables, context lengths)."""

    def __init__(self, num_blocks: int, block_size: int = PA_BLOCK_SIZE):
        self._L = lib()
        self._h = self._L.pa_bm_create(int(num_blocks), int(block_size))
        if not self._h:
            raise PaError(PA_ERR_INVALID_ARG, "pa_bm_create")
        self.num_blocks = int(num_blocks)

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def num_free(self) -> int:
        return int(self._L.pa_bm_num_free_blocks(self._h))

    def add_sequence(self, seq_id: int, num_tokens: int) -> None:
        _check(self._L.pa_bm_add_sequence(self._h, int(seq_id), int(num_tokens)), "pa_bm_add_sequence")

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(self._L.pa_bm_fork(self._h, int(parent_id), int(child_id)), "pa_bm_fork")

    def free(self, seq_id: int) -> None:
        _check(self._L.pa_bm_free_sequence(self._h, int(seq_id)), "pa_bm_free_sequence")

    def slots(self, seq_id: int, start: int, count: int):
        import numpy as np
        out = np.empty(max(int(count), 0), dtype=np.int64)
        _check(self._L.pa_bm_slots(self._h, int(seq_id), int(start), int(count),
                                   out.ctypes.data if count > 0 else None), "pa_bm_slots")
        return out

    def append_slots(self, seq_ids):
        """Reserve the next token's slot of each sequence. Returns
        (slot_mapping int64 [n], cow_pairs int64 [k, 2])."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.empty(n, dtype=np.int64)
        cow = np.empty((max(n, 1), 2), dtype=np.int64)
        nc = ctypes.c_int32(0)
        _check(self._L.pa_bm_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                          cow.ctypes.data, ctypes.byref(nc)), "pa_bm_append_slots")
        return slots, cow[:nc.value].copy()

    def block_tables(self, seq_ids, stride: int):
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        bt = np.empty((ids.size, int(stride)), dtype=np.int32)
        lens = np.empty(ids.size, dtype=np.int32)
        _check(self._L.pa_bm_block_tables(self._h, ids.ctypes.data, ids.size, bt.ctypes.data,
                                          int(stride), lens.ctypes.data), "pa_bm_block_tables")
        return bt, lens

    def stats(self) -> dict:
        st = _BmStats()
        _check(self._L.pa_bm_get_stats(self._h, ctypes.byref(st)), "pa_bm_get_stats")
        return {n: int(getattr(st, n)) for n, _ in _BmStats._fields_}

    def refcount(self, block: int) -> int:
        return int(self._L.pa_bm_refcount(self._h, int(block)))
