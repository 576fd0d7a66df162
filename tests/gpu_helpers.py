"""Shared helpers for the GPU tests: move a workload to the device, run the
step through libpa, run the same step through the oracle, compare."""
import numpy as np
import torch

import oracle
from paged_kv_cache_391_b200 import pa

# Tolerance of pa_decode against the fp64 oracle: max |gpu - ref| <= 2e-2 over
# all elements, and per (sequence, head) row max|gpu - ref| / max|ref| <= 1e-2.
MAX_ABS = 2e-2
ROW_REL = 1e-2


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float16


def dev16(a: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype).cuda()


def host16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class DeviceStep:
    """The workload's buffers on the device and one step through libpa."""

    def __init__(self, w, partition_tokens=None):
        self.w = w
        dt = torch_dtype(w)
        self.dt = dt
        self.k_cache = dev16(w.k_pool, dt)
        self.v_cache = dev16(w.v_pool, dt)
        self.q = dev16(w.q, dt)
        self.new_k = dev16(w.new_k, dt)
        self.new_v = dev16(w.new_v, dt)
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.pairs = torch.from_numpy(w.copy_pairs).cuda()
        self.bt = torch.from_numpy(w.block_tables).cuda()
        self.cl = torch.from_numpy(w.context_lens).cuda()
        self.out = torch.empty(w.q.shape, dtype=dt, device="cuda")
        self.P = w.partition_tokens if partition_tokens is None else partition_tokens
        self.ws = pa.alloc_workspace(int(w.q.shape[0]), w.num_q_heads, w.head_dim,
                                     w.max_context_len, self.P, "cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def cache_ops(self):
        if self.pairs.numel():
            pa.copy_blocks([self.k_cache], [self.v_cache], self.pairs, dev_error=self.err)
        pa.write_kv(self.new_k, self.new_v, self.k_cache, self.v_cache, self.slots,
                    dev_error=self.err)

    def decode(self, out=None):
        out = self.out if out is None else out
        pa.decode(out, self.q, self.k_cache, self.v_cache, self.bt, self.cl, scale=self.w.scale,
                  max_context_len=self.w.max_context_len, partition_tokens=self.P,
                  workspace=self.ws, dev_error=self.err)
        return out

    def prefill(self, out=None, ordered=False):
        """The chunk attention of a workload built by workloads.chunk_workload.
        ordered=True gives pa_prefill_chunk the larger workspace of
        pa_prefill_chunk_workspace_size, with which the tcgen05 path runs its
        work longest first (a plan kernel); otherwise the partials' workspace
        only (grid order)."""
        out = self.out if out is None else out
        w = self.w
        qs = torch.from_numpy(w.q_start).cuda()
        mq = int(np.diff(w.q_start).max())
        ws = self.ws
        if ordered:
            ws = pa.alloc_chunk_workspace(int(w.q.shape[0]), w.num_seqs, w.num_q_heads,
                                          w.group_size, w.head_dim, mq, w.max_context_len,
                                          self.P, "cuda")
        pa.prefill_chunk(out, self.q, qs, self.k_cache, self.v_cache, self.bt, self.cl,
                         scale=w.scale, max_query_len=mq, max_context_len=w.max_context_len,
                         partition_tokens=self.P, workspace=ws, dev_error=self.err)
        return out

    def step(self):
        self.cache_ops()
        self.decode()
        torch.cuda.synchronize()
        return self


def oracle_caches_after_step(w):
    kc, vc = w.k_pool.copy(), w.v_pool.copy()
    if len(w.copy_pairs):
        oracle.copy_blocks([kc], [vc], w.copy_pairs)
    assert oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping) == 0
    return kc, vc


def assert_decode_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    """gpu, ref: [..., D] float64 arrays of the same shape."""
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    row_err = err.reshape(-1, ref.shape[-1]).max(axis=1)
    row_ref = np.abs(ref).reshape(-1, ref.shape[-1]).max(axis=1)
    rel = row_err / np.maximum(row_ref, 1e-6)
    assert rel.max() <= ROW_REL, f"{what}: max row rel err {rel.max():.3e} at row {rel.argmax()}"
    return err.max(), rel.max()
