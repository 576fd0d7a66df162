"""Host-side pieces of bench.py that need no GPU: input packing for the
end-to-end path, L2 notes, the CPU (oracle) leg on a tiny workload."""
import numpy as np
import torch

import bench
from paged_kv_cache_391_b200 import workloads as W


def test_packed_inputs_round_trip():
    for w in (W.tiny(), W.shared_prefix(num_seqs=3, prefix=100, suffix_hi=30)):
        dt = torch.float16 if w.dtype == "f16" else torch.bfloat16
        p = bench.PackedInputs(w, dt, pin=False)
        assert p.nbytes % 256 == 0
        assert p.payload == sum(a.nbytes for a in (w.q, w.new_k, w.new_v, w.slot_mapping,
                                                     w.copy_pairs, w.block_tables, w.context_lens))
        v = p.views(p.host.clone())
        assert np.array_equal(v["q"].view(torch.int16).numpy().view(np.uint16), w.q)
        assert np.array_equal(v["new_v"].view(torch.int16).numpy().view(np.uint16), w.new_v)
        assert np.array_equal(v["slots"].numpy(), w.slot_mapping)
        assert np.array_equal(v["pairs"].numpy(), w.copy_pairs)
        assert np.array_equal(v["bt"].numpy(), w.block_tables)
        assert np.array_equal(v["cl"].numpy(), w.context_lens)
        for name, (off, *_rest) in p.layout.items():
            assert off % 256 == 0, name


def test_l2_notes():
    assert bench.l2_note(W.shared_prefix(num_seqs=5, prefix=400, suffix_hi=40)).startswith("shared")
    assert "within 2x" in bench.l2_note(W.mha(batch=2))


def test_cpu_leg_on_tiny():
    r = bench.oracle_sample(W.tiny(), 0.05)
    assert r["gbs"] > 0 and r["cores"] >= 1 and "rows" in r["sample"]
