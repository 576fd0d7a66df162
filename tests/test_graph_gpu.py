"""A decode step captured once as a CUDA graph and replayed.

libpa's calls only launch kernels on the caller's stream (their host-side
work -- argument checks, tensor-map encoding, occupancy queries -- makes no
stream operation), so a whole step (copy-on-write copies, KV write, attention
with its plan and reduce kernels, programmatic dependent launches included)
can be captured into a graph and replayed without the per-call host cost.
The replay must give the eager step's bits, and must read the buffers' current
contents: new queries written between replays give the new result."""
import numpy as np
import pytest
import torch

from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import DeviceStep, dev16

pytestmark = pytest.mark.gpu


def _make(mode):
    if mode == "chunk":
        w = W.chunked_prefill(batch=3, chunk=128)
        d = DeviceStep(w)
        mq = int(np.diff(w.q_start).max())
        ws = pa.alloc_chunk_workspace(int(w.q.shape[0]), w.num_seqs, w.num_q_heads, w.group_size,
                                      w.head_dim, mq, w.max_context_len, d.P, "cuda")
        qs = torch.from_numpy(w.q_start).cuda()

        def attend(out):
            pa.prefill_chunk(out, d.q, qs, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
                             max_query_len=mq, max_context_len=w.max_context_len,
                             partition_tokens=d.P, workspace=ws, dev_error=d.err)
        return w, d, attend
    if mode == "shared":
        w = W.shared_prefix(num_seqs=24, prefix=2100, suffix_hi=300)
        d = DeviceStep(w, 512)
        ws = pa.alloc_workspace(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len, 512,
                                "cuda")
        shared = int(w.notes["shared_blocks"]) * pa.PA_BLOCK_SIZE

        def attend(out):
            pa.decode(out, d.q, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
                      max_context_len=w.max_context_len, partition_tokens=512, workspace=ws,
                      dev_error=d.err, shared_prefix_tokens=shared)
        return w, d, attend
    w = W.tiny() if mode == "tiny" else W.gqa(batch=12)
    d = DeviceStep(w, partition_tokens=16 if mode == "tiny" else None)
    persistent = mode == "persistent"
    ws = pa.alloc_workspace(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len, d.P,
                            "cuda", persistent=persistent)

    def attend(out):
        pa.decode(out, d.q, d.k_cache, d.v_cache, d.bt, d.cl, scale=w.scale,
                  max_context_len=w.max_context_len, partition_tokens=d.P, workspace=ws,
                  dev_error=d.err, persistent=persistent)
    return w, d, attend


@pytest.mark.parametrize("mode", ["tiny", "grid", "persistent", "chunk", "shared"])
def test_step_replays_as_a_cuda_graph(mode):
    w, d, attend = _make(mode)

    def step(out):
        d.cache_ops()     # copy-on-write copies (tiny) and the KV write
        attend(out)

    eager = torch.empty_like(d.out)
    step(eager)
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graphed = torch.full_like(d.out, float("nan"))
    with torch.cuda.stream(s):       # first calls outside the capture
        step(graphed)
    torch.cuda.synchronize()
    graphed.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(graphed)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(graphed.view(torch.int16), eager.view(torch.int16))

    # the replay reads the buffers as they are now: new queries, new result
    rng = np.random.default_rng(5)
    q2 = W._normal_bits(rng, w.q.shape, w.dtype)
    d.q.copy_(dev16(q2, d.dt))
    g.replay()
    torch.cuda.synchronize()
    eager2 = torch.empty_like(d.out)
    step(eager2)
    torch.cuda.synchronize()
    assert torch.equal(graphed.view(torch.int16), eager2.view(torch.int16))
    assert not torch.equal(eager2.view(torch.int16), eager.view(torch.int16))
    assert int(d.err.item()) == 0
