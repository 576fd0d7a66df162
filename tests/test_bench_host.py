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


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints
    one JSON line with the keys the driver reads, on a bounded sample."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=300,
                       cwd=root)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] == d["e2e"]["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_0_only():
    """Launched by torchrun with N > 1, the reference arm's other ranks exit 0
    at once and print nothing (rank 0 alone times the oracle)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=300,
                       cwd=root, env=env)
    assert r.returncode == 0, r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_recorded_traffic_follows_the_kernel_sources():
    """A traffic figure is reported for a full-size workload only while the
    hash of its kernel family's sources matches the recorded one."""
    assert bench.recorded_traffic("mha", batch=16) is None        # not the full size
    assert bench.recorded_traffic("no_such_workload", None) is None
    fam = {"chunked_prefill": "tcgen05", "mha": "mma"}
    with open(bench.TRAFFIC_FILE) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for key, h, nbytes, alg, ratio in rows:
        workload, _, sched = key.partition(":")
        want = bench.kernel_source_hash("tcgen05" if workload in bench.TC_WORKLOADS else "mma")
        got = bench.recorded_traffic(workload, None, sched or "grid")
        assert got == (int(nbytes) if h == want else None), key
        assert abs(int(nbytes) / int(alg) - float(ratio)) < 1e-3
    assert set(fam) <= {r[0].partition(":")[0] for r in rows}


def _reached(w):
    used = set()
    for s, L in enumerate(w.context_lens):
        used.update(int(b) for b in w.block_tables[s, :W.blocks_needed(int(L))])
    return used


def test_timed_block_copies_never_touch_the_step_cache():
    """The copies timed on their own: the step's forks when it has any, else
    copies into blocks that no table reaches (so the timed loop leaves the
    decode's cache as it was)."""
    w = W.tiny()
    pairs, what = bench.timing_copy_pairs(w)
    assert np.array_equal(pairs, w.copy_pairs) and "step" in what
    for w in (W.shared_prefix(num_seqs=5, prefix=300, suffix_hi=40), W.mha(batch=4)):
        pairs, _ = bench.timing_copy_pairs(w)
        reached = _reached(w)
        assert len(pairs) == w.num_seqs
        assert not set(pairs[:, 1].tolist()) & reached
        assert len(set(pairs[:, 1].tolist())) == len(pairs)
        assert set(pairs[:, 0].tolist()) <= reached | {w.notes.get("partial_prefix_block", -1)}
    forks = np.asarray(w.notes.get("fork_pairs", []))
    assert forks.size == 0   # mha has no forks: the timed copies fork each last block


def test_last_block_waste():
    """Waste = the unused tail of each last block: lengths 16, 17, 31, 1 leave
    0, 15, 1 and 15 slots of 16, 32, 32 and 16 allocated."""
    w = W.tiny()
    w.context_lens = np.array([16, 17, 31, 1], np.int32)
    r = bench.waste_stats(w)
    assert r["mean_slots_per_seq"] == 7.75
    assert r["pct_of_allocated_slots"] == round(100 * 31 / 96, 4)


def test_shared_prefix_record_counts_the_shared_partitions_once():
    """The bench record of the shared-prefix path (synthetic timings, no GPU):
    the roofline's bytes are the distinct K/V bytes (9 shared partitions of
    512 tokens once, the rest per sequence); the logical rate stays in
    kv_gbs; the record is plain JSON."""
    import argparse
    import json
    w = bench.make_workload("shared_prefix", None)
    res = {"w": w, "sus_reps": 10, "persistent": False, "shared_tokens": 4992, "tc_path": False,
           "copy_pairs": 0, "copy_what": "", "short_reps": 200, "rounds": 1, "launches": 4,
           "e2e": None, "att_reps": 20}
    agg = {"ms": 1.3, "att_ms": 0.06, "kv": w.kv_bytes(), "sus_ms": 0.07, "seqs": w.num_seqs,
           "write_ms": 0.004, "copy_ms": 0.004, "errors": 0, "e2e_ms": 1.4}
    args = argparse.Namespace(steps=20, batch=None, workload="long", sustain_seconds=3.0,
                              scheduler="shared")
    ceiling = {"gbs": 7100.0, "scattered_tiles_gbs": 6800.0, "bytes": 2 << 30,
               "vector_loads_gbs": 7000.0, "bulk_copies_gbs": 7100.0}
    rec = bench.workload_record("shared_prefix", res, agg, args, 1, ceiling)
    roof = rec["roofline"]
    per_seq = 9 * 512 * w.num_kv_heads * w.head_dim * 2 * 2
    distinct = w.step_bytes()["decode"] - (w.num_seqs - 1) * per_seq
    assert roof["algorithmic_bytes_per_launch"] == distinct
    assert abs(roof["achieved"] - distinct / 0.06e-3 / 1e9) < 0.1
    assert roof["kv_gbs"] > 5 * roof["achieved"]          # logical: every whole context
    assert roof["bound"] == "hbm" and roof["traffic"] is None
    assert "pa_decode_shared_prefix" in roof["kernel"]
    json.dumps(rec)
