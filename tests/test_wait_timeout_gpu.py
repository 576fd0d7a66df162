"""The bounded-wait timeout path of the decode kernel, made to run out
without withholding anything from the GPU.

A test-only build of libpa (``build.build_variant("waittest")``, compiled with
PA_TEST_TILE_WAIT_EXPIRED) makes every K/V tile wait of the decode kernels
report at once that it ran out of time, as a real wait does after its limit.
What follows is the product code path unchanged: the warp waits (bounded, the
full limit) for the copies it has in flight, adds PA_DEV_ERR_TIMEOUT to
dev_error, and the CTA merges what it has and returns. Every copy is a valid
in-bounds load that completes; nothing waits for anything that is never
coming.

The checks: the call returns normally, every warp with a tile reported one
timeout and nothing else was counted, each warp gave up before its first tile
so the output is exactly zero (an empty softmax), the CUDA context stays
usable, and the product library's next decode on the same device matches the
oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_391_b200 import build as pa_build
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, assert_decode_close, oracle_caches_after_step, to_f64
import oracle

pytestmark = pytest.mark.gpu


def _waittest_lib():
    L = ctypes.CDLL(pa_build.build_variant("waittest"))
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.pa_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, i32,
                            ctypes.c_float, i32, P, sz, P, ctypes.c_int, P]
    L.pa_decode.restype = ctypes.c_int
    return L


def test_tile_wait_that_runs_out_is_reported_and_leaves_the_context_usable():
    # 2 sequences x 2 KV heads, 4096 tokens, no split: 4 CTAs of 4 warps, each
    # warp with 64 tiles and two copies in flight when its first wait gives
    # up; 16 timeouts of 2^24 each stay within int32.
    w = W.decode_workload("waittest", [4096, 4096], num_q_heads=2, num_kv_heads=2,
                          head_dim=128, dtype="bf16", seed=11, partition_tokens=0)
    d = DeviceStep(w, partition_tokens=0)
    d.cache_ops()
    torch.cuda.synchronize()
    L = _waittest_lib()
    out = torch.zeros_like(d.out)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.pa_decode(out.data_ptr(), d.q.data_ptr(), d.k_cache.data_ptr(), d.v_cache.data_ptr(),
                     d.bt.data_ptr(), d.bt.shape[1], d.cl.data_ptr(), w.num_seqs, w.num_q_heads,
                     w.group_size, w.head_dim, pa.PA_BLOCK_SIZE, w.num_blocks, w.max_context_len,
                     ctypes.c_float(w.scale), 0, None, 0, err.data_ptr(), pa.PA_DTYPE_BF16,
                     torch.cuda.current_stream().cuda_stream)
    assert st == pa.PA_OK
    torch.cuda.synchronize()                    # the kernel returned; the context answers
    e = int(err.item())
    assert e == 16 * pa.PA_DEV_ERR_TIMEOUT, hex(e)   # one per warp, no data error
    assert torch.equal(out, torch.zeros_like(out))   # no key was taken: zeros, no NaN

    # the product library on the same context and data: the oracle's result
    kc, vc = oracle_caches_after_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype)
    d.decode()
    torch.cuda.synchronize()
    assert_decode_close(to_f64(d.out), ref, "product decode after the timeout test")
    assert int(d.err.item()) == 0
