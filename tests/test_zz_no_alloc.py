"""pa_decode_static: decode attention for callers that may not allocate
device memory.

Some callers cannot call cudaMalloc: a plugin living inside a host
application that owns all device memory and forbids its plugins from
allocating, or a decode loop where cudaMalloc/cudaFree (which can synchronise
the whole device) are not acceptable. pa_decode_static serves them with a
fixed scratch array compiled into libpa instead of a caller workspace. These
tests call it through the C ABI and check that, on calls made back to back
(the scratch keeps the previous call's contents), it gives bit for bit what
pa_decode gives with a caller workspace -- the same kernels on the same
inputs -- and the oracle's result within the decode tolerance; and that
sizes beyond the array are refused before anything is launched.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, assert_decode_close, oracle_caches_after_step, to_f64

pytestmark = pytest.mark.gpu


def _static_call(d, out):
    """pa_decode_static straight through ctypes, no workspace argument."""
    w = d.w
    return pa.lib().pa_decode_static(
        out.data_ptr(), d.q.data_ptr(), d.k_cache.data_ptr(), d.v_cache.data_ptr(),
        d.bt.data_ptr(), d.bt.shape[1], d.cl.data_ptr(), w.num_seqs, w.num_q_heads,
        w.group_size, w.head_dim, pa.PA_BLOCK_SIZE, w.num_blocks, w.max_context_len,
        ctypes.c_float(w.scale), d.P, d.err.data_ptr(),
        pa.PA_DTYPE_BF16 if w.dtype == "bf16" else pa.PA_DTYPE_F16,
        torch.cuda.current_stream().cuda_stream)


def test_static_scratch_matches_caller_workspace_on_calls_in_a_row():
    a = DeviceStep(W.mha(batch=6))
    b = DeviceStep(W.gqa(batch=10))
    for d in (a, b, a):   # back to back: each call finds the previous call's partials
        w = d.w
        need = pa.decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim,
                                        w.max_context_len, d.P)
        assert 0 < need <= pa.PA_STATIC_WORKSPACE_BYTES   # the split-K path is exercised
        d.cache_ops()
        ref = d.decode().clone()                            # caller-provided workspace
        out = torch.full_like(ref, float("nan"))
        assert _static_call(d, out) == pa.PA_OK
        torch.cuda.synchronize()
        # same kernels, same inputs, same partition size: the same bits
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert int(d.err.item()) == 0
    # and the result is the oracle's, within the decode tolerance
    kc, vc = oracle_caches_after_step(a.w)
    want = oracle.decode(a.w.q, kc, vc, a.w.block_tables, a.w.context_lens, a.w.scale,
                         a.w.dtype)
    assert_decode_close(to_f64(out), want, "pa_decode_static vs oracle")


def test_sizes_beyond_the_static_scratch_are_refused():
    # A launch whose partials would not fit: 4096 sequences x 64 heads x 256
    # partitions. No buffer is passed at all, so even a check order that
    # regressed could not launch anything (it would return
    # PA_ERR_INVALID_ARG instead of the size status asserted here).
    need = pa.decode_workspace_size(4096, 64, 128, 131072, 512)
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    st = pa.lib().pa_decode_static(
        None, None, None, None, None, 8192, None, 4096, 64, 8, 128, 16, 1 << 20,
        131072, ctypes.c_float(0.088), 512, None, pa.PA_DTYPE_BF16,
        torch.cuda.current_stream().cuda_stream)
    assert st == pa.PA_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
