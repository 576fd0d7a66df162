#!/usr/bin/env python
"""Benchmark of the paged decode step on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic input:
copy-on-write block copies (when the workload forks blocks), the KV write of
this step's tokens, and paged decode attention (partition kernel plus the
log-sum-exp reduce when a context spans several partitions), all through
libpa's C ABI on the current CUDA stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mha|gqa|shared_prefix|long|...]
                  [--scheduler grid|persistent|shared]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed on the host cores

Multi-GPU (launched by torch.distributed.run): every rank runs its own
independent workload (sequences are independent), so per-GPU work is fixed
(weak scaling); the only collectives are a barrier and a max/sum of timings.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode KV GB/s & fraction of B200 HBM peak; seq-steps/s at 1 GPU"
L2_BYTES = 126_000_000
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_TEXT = {
    "tiny": "tiny: 4+1 seqs, ctx {8,17,34,51,51}, H_q=H_kv=4, D=64, fp16, 32-block pool, 1 CoW fork",
    "mha": "Llama-2-7B-shaped MHA decode, 1 layer: batch 64, H_q=H_kv=32, D=128, fp16, "
           "block 16, ctx U[128,2048], pool 1.5x needed",
    "gqa": "Llama-3-8B-shaped GQA decode, 1 layer: batch 256, H_q=32, H_kv=8, D=128, bf16, "
           "block 16, ctx lognormal(median 1024, sigma 1) clipped [16,8192]",
    "shared_prefix": "shared-prefix decode: 100 seqs sharing a 5000-token prefix (312 full blocks + "
                     "1 partial CoW-forked per seq), suffix U[16,512], H_q=32, H_kv=8, D=128, bf16",
    "long": "long-context 70B-shaped GQA decode, 1 layer: batch 8, H_q=64, H_kv=8, D=128, bf16, "
            "ctx U[32768,131072], split-K 512-token partitions + LSE reduce",
    "spec_verify": "speculative verify on the Llama-3-8B GQA batch: 256 seqs, 4 draft tokens each "
                   "(causal in the chunk), H_q=32, H_kv=8, D=128, bf16, ctx lognormal(1024, 1), "
                   "2048-token partitions",
    "chunked_prefill": "chunked prefill, Llama-3-8B shape: 16 prompts of U[1024,8192] tokens, "
                       "next 256-token chunk each, H_q=32, H_kv=8, D=128, bf16",
    "skewed": "skewed-length decode, Llama-3-8B GQA shape: batch 256, 4 contexts U[65536,131072] "
              "among 252 lognormal(median 512, sigma 0.7) clipped [16,4096], H_q=32, H_kv=8, "
              "D=128, bf16, 2048-token partitions",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long", choices=list(WORKLOAD_TEXT),
                    help="the headline workload (default: the long-context config, the "
                         "largest that fits one GPU)")
    ap.add_argument("--also", default="gqa,chunked_prefill,shared_prefix:shared",
                    help="comma-separated workloads measured in the same run and reported "
                         "under 'also' (empty: none); workload:scheduler picks that "
                         "workload's scheduler")
    ap.add_argument("--batch", type=int, default=None, help="override the batch (profiling only)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="step", choices=["step", "swap", "blockmgr"],
                    help="step: the decode step (default); swap: preemption swap-out/in; "
                         "blockmgr: host block-manager throughput (no GPU)")
    ap.add_argument("--partition-tokens", type=int, default=None)
    ap.add_argument("--scheduler", default="grid", choices=["grid", "persistent", "shared"],
                    help="decode schedule: grid = pa_decode (one CTA per partition); "
                         "persistent = pa_decode_persistent (plan + work queue); shared = "
                         "pa_decode_shared_prefix for the shared_prefix workload (the shared "
                         "partitions as one tcgen05 contraction over all sequences)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--op-seconds", type=float, default=0.6,
                    help="target GPU time of the write_kv and copy_blocks timing loops")
    ap.add_argument("--sustain-seconds", type=float, default=3.0,
                    help="GPU time of the sustained attention loop (power-capped clocks)")
    ap.add_argument("--no-read-probe", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle sample")
    return ap.parse_args()


def make_workload(name, batch, seed_offset=0):
    from paged_kv_cache_391_b200 import workloads as W
    kw = {}
    if batch is not None:
        kw["num_seqs" if name == "shared_prefix" else "batch"] = batch
    fn = W.CONFIGS[name]
    import inspect
    seed = inspect.signature(fn).parameters["seed"].default + 1000 * seed_offset
    return fn(seed=seed, **kw)


# The sources each kernel family is built from: a recorded traffic figure is
# valid only while the hash of its family's sources is unchanged.
KERNEL_SOURCES = {
    "mma": ("paged_kv_cache_391_b200/csrc/pa_decode.cu",
            "paged_kv_cache_391_b200/csrc/pa_device.cuh"),
    "tcgen05": ("paged_kv_cache_391_b200/csrc/pa_prefill_tc.cu",
                "paged_kv_cache_391_b200/csrc/pa_tcgen05.cuh",
                "paged_kv_cache_391_b200/csrc/pa_device.cuh"),
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
TC_WORKLOADS = ("chunked_prefill",)  # the configs whose chunks take the tcgen05 kernel


def kernel_source_hash(family: str = "mma") -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[family]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, batch, scheduler: str = "grid"):
    """DRAM bytes (read + write) per attention call from the ncu capture
    recorded in profiles/dram_traffic.txt for this workload, or None when
    there is none or its kernel sources changed since it was taken."""
    if batch is not None or not os.path.exists(TRAFFIC_FILE):
        return None
    want = kernel_source_hash("tcgen05" if workload in TC_WORKLOADS else "mma")
    key = workload if scheduler == "grid" else f"{workload}:{scheduler}"
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split("#")[0].split()
            if len(parts) >= 3 and parts[0] == key and parts[1] == want:
                return int(parts[2])
    return None


FALLBACK_BF16_TFLOPS = 1590.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak(sustained: bool = False):
    """Dense bf16 tensor peak (TFLOP/s): the burst figure for a kernel timed
    in short loops, the sustained one (seconds under the power cap) for the
    sustained loop; fp16 has the same nominal rate."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if key in d:
            return float(d[key]), f"measured (MEASURED_PEAKS.json {key})"
    return (1400.0 if sustained else FALLBACK_BF16_TFLOPS), "fallback"


def attention_flops(w) -> float:
    """Multiply-adds of q.K and P.V: 4 * D flops per (query row, head, key seen)."""
    L = w.context_lens.astype(np.int64)
    if w.q_start is None:
        keys = L.sum()
    else:
        tq = np.diff(w.q_start).astype(np.int64)
        # query t of a chunk of tq at the end of L sees L - tq + t + 1 keys
        keys = int((tq * (L - tq) + tq * (tq + 1) // 2).sum())
    return 4.0 * w.head_dim * w.num_q_heads * float(keys)


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) while
    the timed region runs."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index: int, interval_s: float = 0.001):
        self.interval = interval_s
        self.samples, self.reasons, self.err = [], set(), None
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.nv, self.err = None, f"nvml unavailable: {e}"

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, const in self.REASONS.items():
                    if r & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
            time.sleep(self.interval)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_min_mhz": min(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples),
                "how": f"NVML every {self.interval * 1e3:g} ms across every timed loop (the K "
                       f"steps, the per-operation loops, the read-ceiling probe, e2e)"}


# --------------------------------------------------------------------------- CPU (oracle) leg

def oracle_sample(w, target_s: float):
    """Time the fp64 CPU oracle on a bounded sample of the step: the whole
    step's cache writes plus decode of a random subset of (sequence, head)
    rows, sized to take about target_s seconds on every host core. Returns the
    step-equivalent KV GB/s, seq-steps/s, cores, and a description."""
    import oracle
    n_rows = w.num_seqs * w.num_q_heads
    cores = oracle.num_cores()
    rng = np.random.default_rng(0)
    kc, vc = w.k_pool.copy(), w.v_pool.copy()

    def run(rows):
        t0 = time.perf_counter()
        if len(w.copy_pairs):
            oracle.copy_blocks([kc], [vc], w.copy_pairs)
        oracle.write_kv(w.new_k, w.new_v, kc, vc, w.slot_mapping)
        oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, w.dtype, rows=rows)
        return time.perf_counter() - t0

    # calibrate on a few rows, then size the sample
    order = rng.permutation(n_rows)
    probe = np.sort(order[:min(n_rows, max(cores, 8))])
    dt = run(probe)
    per_row = dt / len(probe)
    n = int(min(n_rows, max(len(probe), target_s / max(per_row, 1e-9))))
    rows = np.sort(order[:n])
    dt = run(rows)
    reps = 1
    if n == n_rows and dt < target_s:   # the whole step is quick: repeat it up to the target
        reps = max(1, int(target_s / max(dt, 1e-9)))
        dt = sum(run(rows) for _ in range(reps)) / reps
    # step-equivalent work: the sampled rows' share of the decode
    row_bytes = (w.context_lens.astype(np.int64)[rows // w.num_q_heads]).sum() * 2 * \
        w.head_dim * 2 / w.group_size
    frac_seqs = n / n_rows
    return {
        "gbs": row_bytes / dt / 1e9,
        "seq_steps_per_s": frac_seqs * w.num_seqs / dt,
        "seconds": dt, "cores": cores,
        "sample": f"{n} of {n_rows} (seq, q-head) rows of one step (mean of {reps} runs), with "
                  f"the step's whole write_kv/copy_blocks; KV bytes counted per KV head as on "
                  f"the GPU",
    }


# --------------------------------------------------------------------------- GPU leg

class PackedInputs:
    """A step's inputs (q, new K/V rows, slots, CoW pairs, tables, lengths)
    packed at 256-byte aligned offsets in one buffer, so a whole step's
    inputs cross from pinned host memory in one copy."""

    def __init__(self, w, dt, pin: bool = True):
        import torch
        self.dt = dt
        parts = [("q", w.q.view(np.int16)), ("new_k", w.new_k.view(np.int16)),
                 ("new_v", w.new_v.view(np.int16)), ("slots", w.slot_mapping),
                 ("pairs", w.copy_pairs), ("bt", w.block_tables), ("cl", w.context_lens)]
        if w.q_start is not None:
            parts.append(("q_start", w.q_start))
        self.layout, off = {}, 0
        for name, a in parts:
            a = np.ascontiguousarray(a)
            self.layout[name] = (off, a.dtype, a.shape, a.nbytes)
            off += (a.nbytes + 255) // 256 * 256
        self.nbytes = off
        self.host = torch.empty(off, dtype=torch.uint8)
        if pin:
            self.host = self.host.pin_memory()
        hv = self.host.numpy()
        for name, a in parts:
            o, dtype, shape, n = self.layout[name]
            hv[o:o + n] = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        self.payload = sum(v[3] for v in self.layout.values())

    def views(self, buf):
        """Typed tensor views of a device buffer laid out like the host one."""
        import torch
        tmap = {np.dtype(np.int16): torch.int16, np.dtype(np.int64): torch.int64,
                np.dtype(np.int32): torch.int32}
        out = {}
        for name, (o, dtype, shape, n) in self.layout.items():
            t = buf[o:o + n].view(tmap[np.dtype(dtype)]).view(shape)
            out[name] = t.view(self.dt) if dtype == np.int16 else t
        return out


def spare_blocks(w) -> np.ndarray:
    """Physical blocks no table reaches and no copy reads or writes: targets
    for timing block copies without disturbing the step's cache."""
    used = np.zeros(w.num_blocks, dtype=bool)
    for s, L in enumerate(w.context_lens):
        n = -(-int(L) // w.block_size)
        used[w.block_tables[s, :n]] = True
    for pairs in (w.copy_pairs, np.asarray(w.notes.get("fork_pairs", []), np.int64).reshape(-1, 2)):
        if len(pairs):
            used[pairs.reshape(-1)] = True
    return np.flatnonzero(~used)


def timing_copy_pairs(w):
    """The block copies timed on their own, and what they are: the config's
    copy-on-write forks when it has any (into spare blocks when the fork
    happened before the step), else a fork of every sequence's last block
    into a spare block (the cost of forking each sequence once)."""
    spare = spare_blocks(w)
    if len(w.copy_pairs):
        return w.copy_pairs, "the step's copy-on-write forks"
    forks = np.asarray(w.notes.get("fork_pairs", []), np.int64).reshape(-1, 2)
    if len(forks):
        n = min(len(forks), len(spare))
        return (np.stack([forks[:n, 0], spare[:n]], axis=1).astype(np.int64),
                f"the config's {n} copy-on-write forks of the partial prefix block "
                f"(made before the step; timed into spare blocks)")
    last = np.array([w.block_tables[s, max(0, -(-int(L) // w.block_size) - 1)]
                     for s, L in enumerate(w.context_lens)], np.int64)
    n = min(len(last), len(spare))
    return (np.stack([last[:n], spare[:n]], axis=1).astype(np.int64),
            f"a fork of each of {n} sequences' last block into a spare block "
            f"(the config's step copies nothing)")


def waste_stats(w) -> dict:
    """Slots allocated but not holding a token: the unused tail of each
    sequence's last block (the only waste of 16-token paging)."""
    L = w.context_lens.astype(np.int64)
    alloc = -(-L // w.block_size) * w.block_size
    waste = alloc - L
    return {"mean_slots_per_seq": round(float(waste.mean()), 3),
            "pct_of_allocated_slots": round(100.0 * float(waste.sum()) / float(alloc.sum()), 4)}


def read_ceiling(device, nbytes: int = 2 << 30, reps: int = 10) -> dict:
    """The GPU's streaming-read ceiling (pa_read_probe, both methods): best of
    `reps` timed passes over a buffer of `nbytes` (16x the L2)."""
    import torch
    from paged_kv_cache_391_b200 import pa
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    sink = torch.zeros(1, dtype=torch.int64, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    out = {"bytes": nbytes}
    for method, name in ((0, "vector_loads_gbs"), (1, "bulk_copies_gbs"),
                         (2, "scattered_tiles_gbs")):
        for _ in range(3):
            pa.read_probe(buf, sink, method=method, dev_error=err)
        best = None
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            pa.read_probe(buf, sink, method=method, dev_error=err)
            b.record()
            b.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        moved = nbytes if method < 2 else (nbytes // 8192) * 8192
        out[name] = round(moved / (best / 1e3) / 1e9, 1)
    out["gbs"] = max(out["vector_loads_gbs"], out["bulk_copies_gbs"])
    out["device_errors"] = int(err.item())
    del buf
    return out


def time_loop(fn, reps: int, stream, blocker=None) -> float:
    """Average ms per call of `reps` back-to-back calls of fn on `stream`,
    timed by events at the two ends of the loop. For calls shorter than their
    host-side launch, `blocker` first queues enough GPU work that every call
    is queued before the GPU reaches the first event."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if blocker is not None:
        blocker()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / reps


def run_gpu(args, name, rank, world, device, probe_buf=None, e2e_on=True):
    """One workload on this rank: the K-step timed region, then each
    operation of the step in its own loop, then the end-to-end run."""
    import torch
    from paged_kv_cache_391_b200 import pa

    w = make_workload(name, args.batch if name == args.workload else None, seed_offset=rank)
    if args.partition_tokens is not None:
        w.partition_tokens = args.partition_tokens
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16

    def dev16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).to(device)

    k_cache, v_cache = dev16(w.k_pool), dev16(w.v_pool)
    packed = PackedInputs(w, dt)
    resident = torch.empty(packed.nbytes, dtype=torch.uint8, device=device)
    resident.copy_(packed.host)
    inp = packed.views(resident)
    out = torch.empty(w.q.shape, dtype=dt, device=device)
    P = w.partition_tokens
    n_q = int(w.q.shape[0])
    persistent = args.scheduler == "persistent" and w.q_start is None
    shared_tokens = (int(w.notes["shared_blocks"]) * 16
                     if args.scheduler == "shared" and w.q_start is None
                     and "shared_blocks" in w.notes else 0)
    max_q0 = int(np.diff(w.q_start).max()) if w.q_start is not None else 1
    tc_path = w.q_start is not None and w.head_dim == 128 and max_q0 * w.group_size >= 64
    if w.q_start is not None:   # room for the chunk path's longest-first plan
        ws = pa.alloc_chunk_workspace(n_q, w.num_seqs, w.num_q_heads, w.group_size, w.head_dim,
                                      max_q0, w.max_context_len, P, device)
    else:
        ws = pa.alloc_workspace(n_q, w.num_q_heads, w.head_dim, w.max_context_len, P, device,
                                persistent=persistent)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    max_ctx = w.max_context_len
    max_q = int(np.diff(w.q_start).max()) if w.q_start is not None else 1
    max_parts = 1 if (P == 0 or max_ctx <= P) else -(-max_ctx // P)
    launches_per_step = (1 if len(w.copy_pairs) else 0) + (1 if len(w.slot_mapping) else 0) + \
        1 + (1 if max_parts > 1 else 0) + (1 if persistent else 0) + (1 if tc_path else 0) + \
        (1 if shared_tokens else 0)
    copy_pairs_t, copy_what = timing_copy_pairs(w)
    copy_pairs_dev = torch.from_numpy(copy_pairs_t).to(device)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def copies(x):
        if x["pairs"].numel():
            pa.copy_blocks([k_cache], [v_cache], x["pairs"], dev_error=err, stream=stream)

    def write(x):
        pa.write_kv(x["new_k"], x["new_v"], k_cache, v_cache, x["slots"], dev_error=err,
                    stream=stream)

    def attend(x, o):
        if "q_start" in x:
            pa.prefill_chunk(o, x["q"], x["q_start"], k_cache, v_cache, x["bt"], x["cl"],
                             scale=w.scale, max_query_len=max_q, max_context_len=max_ctx,
                             partition_tokens=P, workspace=ws, dev_error=err, stream=stream)
        else:
            pa.decode(o, x["q"], k_cache, v_cache, x["bt"], x["cl"], scale=w.scale,
                      max_context_len=max_ctx, partition_tokens=P, workspace=ws, dev_error=err,
                      stream=stream, persistent=persistent, shared_prefix_tokens=shared_tokens)

    def step(x, o):
        copies(x)
        write(x)
        attend(x, o)

    def settle():
        # a short idle before a timed loop: clocks recover from the power cap
        # that a previous loop may have reached, so every short loop starts
        # from the same state
        torch.cuda.synchronize(device)
        time.sleep(0.2)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        step(inp, out)
    barrier()
    t_start, t_end = ev(), ev()
    settle()
    barrier()
    t_start.record(stream)
    for _ in range(args.steps):
        step(inp, out)
    t_end.record(stream)
    barrier()
    elapsed_ms = t_start.elapsed_time(t_end)

    # ---- each operation of the step in its own loop (events at the loop ends only)
    step_ms = elapsed_ms / max(1, args.steps)
    sink = torch.zeros(1, dtype=torch.int64, device=device)

    def blocker():  # ~10 ms of queued GPU work ahead of a loop of short calls
        if probe_buf is None:
            return
        for _ in range(30):
            pa.read_probe(probe_buf, sink, method=0, stream=stream)

    # the attention call alone: loops of K calls (the timed region's length and
    # clock conditions), median of three; then a sustained loop of
    # --sustain-seconds under the power cap, reported beside it
    att_reps = max(20, args.steps)
    for _ in range(3):
        attend(inp, out)
    att_loops = []
    for _ in range(3):
        settle()
        att_loops.append(time_loop(lambda: attend(inp, out), att_reps, stream))
    att_ms = float(np.median(att_loops))
    sus_reps = int(min(50000, max(att_reps, args.sustain_seconds / max(att_ms, 1e-3) * 1e3)))
    sus_ms = time_loop(lambda: attend(inp, out), sus_reps, stream)
    short_reps = 200
    rounds = max(1, int(args.op_seconds / 0.012))
    write_ms = min(time_loop(lambda: write(inp), short_reps, stream, blocker)
                   for _ in range(rounds)) if len(w.slot_mapping) else None
    copy_ms = min(time_loop(lambda: pa.copy_blocks([k_cache], [v_cache], copy_pairs_dev,
                                                   dev_error=err, stream=stream),
                            short_reps, stream, blocker)
                  for _ in range(rounds)) if len(copy_pairs_t) else None
    # restore the step's cache state (the copy loop may write over forked blocks)
    step(inp, out)
    torch.cuda.synchronize(device)
    errors = int(err.item())

    # ---- e2e: every step uploads its packed inputs from pinned host memory
    # and reads its output back. Two input/output slots, an upload stream and
    # a download stream let step i+1's upload and step i's download overlap
    # step i's kernels.
    e2e = None
    if e2e_on and not args.no_e2e:
        up_stream, down_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
        dev_in = [torch.empty(packed.nbytes, dtype=torch.uint8, device=device) for _ in range(2)]
        views = [packed.views(b) for b in dev_in]
        outs = [torch.empty_like(out) for _ in range(2)]
        host_out = [torch.empty(out.shape, dtype=dt).pin_memory() for _ in range(2)]
        uploaded = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        downloaded = [torch.cuda.Event() for _ in range(2)]
        started = [False, False]

        def e2e_step(i):
            k = i % 2
            with torch.cuda.stream(up_stream):
                if started[k]:
                    up_stream.wait_event(computed[k])       # slot k's last step has read its inputs
                dev_in[k].copy_(packed.host, non_blocking=True)
                uploaded[k].record(up_stream)
            stream.wait_event(uploaded[k])
            if started[k]:
                stream.wait_event(downloaded[k])            # outs[k] has been read back
            step(views[k], outs[k])
            computed[k].record(stream)
            with torch.cuda.stream(down_stream):
                down_stream.wait_event(computed[k])
                host_out[k].copy_(outs[k], non_blocking=True)
                downloaded[k].record(down_stream)
            started[k] = True

        for i in range(args.warmup):
            e2e_step(i)
        barrier()
        a, b = ev(), ev()
        a.record(stream)
        up_stream.wait_event(a)                             # no upload starts before the clock
        for i in range(args.steps):
            e2e_step(args.warmup + i)
        stream.wait_stream(down_stream)
        b.record(stream)
        barrier()
        e2e = {"ms": a.elapsed_time(b), "h2d": packed.payload,
               "d2h": host_out[0].numel() * host_out[0].element_size()}
    return {"w": w, "elapsed_ms": elapsed_ms, "att_ms": att_ms, "att_reps": att_reps,
            "sus_ms": sus_ms, "sus_reps": sus_reps,
            "write_ms": write_ms, "copy_ms": copy_ms, "copy_pairs": int(len(copy_pairs_t)),
            "copy_what": copy_what, "short_reps": short_reps, "rounds": rounds,
            "errors": errors, "e2e": e2e, "launches": launches_per_step,
            "persistent": persistent, "tc_path": tc_path, "shared_tokens": shared_tokens}


def l2_note(w) -> str:
    """How the step's inputs relate to the 126 MB L2 (no flush between steps)."""
    kv, uniq = w.kv_bytes(), w.unique_kv_bytes()
    if uniq < kv:
        return (f"shared blocks: {kv / 1e6:.0f} MB of logical KV reads per step over "
                f"{uniq / 1e6:.0f} MB of distinct KV; re-reads of shared blocks can hit the "
                f"{L2_BYTES / 1e6:.0f} MB L2, so logical GB/s may exceed the HBM peak")
    if kv > 2 * L2_BYTES:
        return (f"inputs larger than L2: {kv / 1e6:.0f} MB of KV read per step vs "
                f"{L2_BYTES / 1e6:.0f} MB L2, no flush")
    return f"KV per step {kv / 1e6:.0f} MB is within 2x of the {L2_BYTES / 1e6:.0f} MB L2"


def reduce_over_ranks(res, world, device=None):
    """Whole-job figures of one workload: the slowest rank's times (max) and
    every rank's work (sum). One all_reduce each; every rank takes the same
    collective steps."""
    w = res["w"]
    times = [res["elapsed_ms"], res["e2e"]["ms"] if res["e2e"] else 0.0, res["att_ms"],
             res["write_ms"] or 0.0, res["copy_ms"] or 0.0, res.get("sus_ms", 0.0)]
    work = [float(w.kv_bytes()), float(w.num_seqs), float(res["errors"])]
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor(times, dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        s = torch.tensor(work, dtype=torch.float64, device=device)
        dist.all_reduce(s, op=dist.ReduceOp.SUM)
        times, work = t.tolist(), s.tolist()
    return {"ms": float(times[0]), "e2e_ms": float(times[1]), "att_ms": float(times[2]),
            "write_ms": float(times[3]) if res["write_ms"] is not None else None,
            "copy_ms": float(times[4]) if res["copy_ms"] is not None else None,
            "sus_ms": float(times[5]),
            "kv": float(work[0]), "seqs": float(work[1]), "errors": int(work[2])}


def run_swap(args, device):
    """Preemption of half the batch: swap its blocks (K and V, one layer) to a
    pinned host pool and back, timed per direction with CUDA events, next to
    a same-size contiguous pinned copy by the copy engine (the host link's
    ceiling, measured in the same run)."""
    import torch
    from paged_kv_cache_391_b200 import pa
    w = make_workload(args.workload, args.batch)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    kc = torch.from_numpy(w.k_pool.view(np.int16)).view(dt).to(device)
    vc = torch.from_numpy(w.v_pool.view(np.int16)).view(dt).to(device)
    ids = set()
    for s in range(w.num_seqs // 2):
        n = -(-int(w.context_lens[s]) // 16)
        ids.update(int(b) for b in w.block_tables[s, :n])
    ids = sorted(ids)
    n = len(ids)
    shape = (n,) + tuple(kc.shape[1:])
    hk = torch.empty(shape, dtype=dt).pin_memory()
    hv = torch.empty(shape, dtype=dt).pin_memory()
    out_map = torch.tensor([[b, i] for i, b in enumerate(ids)], dtype=torch.int64, device=device)
    in_map = torch.tensor([[i, b] for i, b in enumerate(ids)], dtype=torch.int64, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    nbytes = 2 * hk.numel() * hk.element_size()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def timed(f):
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for _ in range(args.steps):
            f()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    t_out = timed(lambda: pa.swap_blocks([kc], [vc], [hk], [hv], out_map, dev_error=err))
    t_in = timed(lambda: pa.swap_blocks([hk], [hv], [kc], [vc], in_map, dev_error=err))
    dk = torch.empty(shape, dtype=dt, device=device)
    dv = torch.empty(shape, dtype=dt, device=device)
    t_ce_out = timed(lambda: (hk.copy_(dk, non_blocking=True), hv.copy_(dv, non_blocking=True)))
    t_ce_in = timed(lambda: (dk.copy_(hk, non_blocking=True), dv.copy_(hv, non_blocking=True)))
    g = lambda ms: nbytes / (ms / 1e3) / 1e9  # noqa: E731
    line = {
        "metric": "KV block swap GB/s (device <-> pinned host), preemption of half the batch",
        "value": round(2 * nbytes / ((t_out + t_in) / 1e3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "blocks": n, "bytes_per_direction": nbytes,
                   "layers": 1},
        "swap_out_GBs": round(g(t_out), 2), "swap_in_GBs": round(g(t_in), 2),
        "roofline": {"bound": "host link", "peak_out_GBs": round(g(t_ce_out), 2),
                     "peak_in_GBs": round(g(t_ce_in), 2),
                     "peak_source": "contiguous pinned copy of the same bytes by the copy engine, "
                                    "same run",
                     "frac_out": round(t_ce_out / t_out, 4), "frac_in": round(t_ce_in / t_in, 4)},
        "gpu_launches": 2 * args.steps, "device_errors": int(err.item()),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_blockmgr(args):
    """Host time of the block manager's per-step work for a GQA-sized batch:
    256 prompts (lognormal lengths, median 1024), each forked into 4 samples
    (1024 sequences), then `steps` decode steps of append_slots (copy-on-write
    on the first one) + block_tables. The plain-Python model of the same rules
    is timed beside it as the baseline."""
    from oracle.block_manager import BlockManagerModel
    from paged_kv_cache_391_b200 import pa
    rng = np.random.default_rng(7)
    lens = np.clip(np.round(np.exp(np.log(1024.0) + rng.standard_normal(256))), 16, 8192)
    ids = list(range(1024))
    pool = int(sum(-(-int(L) // 16) for L in lens) + 1024 * (args.steps // 16 + 2) + 1024)
    stride = int(-(-(lens.max() + args.steps) // 16)) + 1

    def drive(m, steps):
        for i, L in enumerate(lens):
            m.add_sequence(4 * i, int(L))
            for c in (1, 2, 3):
                m.fork(4 * i, 4 * i + c)
        t0 = time.perf_counter()
        cow = 0
        for _ in range(steps):
            _, c = m.append_slots(ids)
            cow += len(c)
            m.block_tables(ids, stride)
        return (time.perf_counter() - t0) / steps, cow

    native_s, cow = drive(pa.BlockManager(pool), args.steps)
    model_steps = max(1, min(args.steps, 20))
    model_s, _ = drive(BlockManagerModel(pool), model_steps)
    line = {
        "metric": "block-manager host time per decode step (append_slots + block_tables)",
        "value": round(native_s * 1e6, 2), "unit": "us/step", "higher_is_better": False,
        "steps": args.steps, "data": "synthetic",
        "config": {"sequences": len(ids), "prompts": 256, "samples_per_prompt": 4,
                   "prompt_lens": "lognormal(median 1024, sigma 1) clipped [16,8192]",
                   "pool_blocks": pool, "table_stride": stride},
        "cow_copies": cow,
        "seq_steps_per_s": round(len(ids) / native_s, 1),
        "cpu_baseline": {"value": round(model_s * 1e6, 2), "unit": "us/step",
                         "kind": "plain-Python model of the same rules (oracle/block_manager.py)",
                         "steps": model_steps, "cores": 1},
    }
    print(json.dumps(line), flush=True)
    return 0


def kernel_name(w, args) -> str:
    if w.q_start is not None:
        return ("pa_prefill_chunk (chunk_plan_kernel + prefill_tc_kernel on tcgen05 "
                "+ lse_reduce_kernel when split)"
                if int(np.diff(w.q_start).max()) * w.group_size >= 64 else
                "pa_prefill_chunk (decode_partition_kernel + lse_reduce_kernel)")
    if args.scheduler == "persistent":
        return ("pa_decode_persistent (decode_plan_kernel + decode_persistent_kernel + "
                "lse_reduce_kernel)")
    if args.scheduler == "shared" and "shared_blocks" in w.notes:
        return ("pa_decode_shared_prefix (prefill_tc_kernel over the shared partitions of all "
                "sequences on tcgen05 + decode_partition_kernel over the rest + "
                "lse_reduce_kernel)")
    return "pa_decode (decode_partition_kernel + lse_reduce_kernel)"


def workload_record(name, res, agg, args, world, ceiling) -> dict:
    """The figures of one workload: step throughput, the attention call
    against its roofline, each operation's own time, end to end."""
    w = res["w"]
    K = args.steps
    peak, peak_src = measured_peaks()
    tpeak, tpeak_src = measured_tensor_peak()
    sb = w.step_bytes()
    elapsed_ms = agg["ms"]
    att_ms = agg["att_ms"]
    value = agg["kv"] * K / (elapsed_ms / 1e3) / 1e9
    dec_achieved = sb["decode"] / (att_ms / 1e3) / 1e9
    flops = attention_flops(w)
    tensor_bound = flops / (tpeak * 1e12) > sb["decode"] / (peak * 1e9)
    tflops = flops / (att_ms / 1e3) / 1e12
    traffic = recorded_traffic(name, args.batch if name == args.workload else None,
                               args.scheduler)
    roof = {
        "kernel": kernel_name(w, args),
        "bound": "tensor" if tensor_bound else "hbm",
        "achieved": round(tflops, 2) if tensor_bound else round(dec_achieved, 1),
        "peak": tpeak if tensor_bound else peak,
        "peak_source": tpeak_src if tensor_bound else peak_src,
        "unit": "TFLOP/s" if tensor_bound else "GB/s",
        "frac": round(tflops / tpeak, 4) if tensor_bound else round(dec_achieved / peak, 4),
        "kv_gbs": round(dec_achieved, 1),
        "tflops": round(tflops, 2),
        "flops_per_launch": flops,
        "algorithmic_bytes_per_launch": sb["decode"],
        "timing": f"CUDA events at the two ends of a loop of {res['att_reps']} back-to-back "
                  f"attention calls on the launching stream, median of 3 loops (after the "
                  f"{K}-step timed region; max over ranks)",
        "sustained": {
            "achieved": round(flops / (agg["sus_ms"] / 1e3) / 1e12, 2) if tensor_bound
            else round(sb["decode"] / (agg["sus_ms"] / 1e3) / 1e9, 1),
            "frac_of_sustained_peak": round(flops / (agg["sus_ms"] / 1e3) / 1e12 /
                                            measured_tensor_peak(sustained=True)[0], 4)
            if tensor_bound else None,
            "ms": round(agg["sus_ms"], 5), "calls": res["sus_reps"],
            "note": "one loop of back-to-back attention calls lasting about "
                    f"{args.sustain_seconds:g} s (clocks settle under the power cap)"},
        "traffic": traffic,
        "traffic_ratio": round(traffic / sb["decode"], 4) if traffic else None,
        "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the call's "
                        "kernels per call (profiles/dram_traffic.txt; scaled from a reduced "
                        "batch where noted there; null if a kernel source changed since)",
    }
    if ceiling and not tensor_bound:
        roof["peak_read"] = ceiling["gbs"]
        roof["frac_read"] = round(dec_achieved / ceiling["gbs"], 4)
        roof["peak_read_paged"] = ceiling["scattered_tiles_gbs"]
        roof["frac_read_paged"] = round(dec_achieved / ceiling["scattered_tiles_gbs"], 4)
        roof["peak_read_source"] = ("pa_read_probe in this run: best of 10 passes over "
                                    f"{ceiling['bytes'] >> 30} GiB, max of vector loads "
                                    f"({ceiling['vector_loads_gbs']}) and bulk copies "
                                    f"({ceiling['bulk_copies_gbs']}) GB/s; peak_read_paged: "
                                    f"the same buffer as 4 KiB tiles read once each in a "
                                    f"scattered order by 2 KiB TMA boxes in the decode "
                                    f"kernel's CTA shape")
    if traffic and not tensor_bound:
        roof["dram_gbs"] = round(traffic / (att_ms / 1e3) / 1e9, 1)
    shared = res.get("shared_tokens", 0)
    if shared and not tensor_bound:
        # pa_decode_shared_prefix reads the shared partitions' K/V once for all
        # sequences: its roofline figure counts those bytes once (the logical
        # figure, each sequence's whole context, stays in kv_gbs and value)
        P = w.partition_tokens
        parts = -(-w.max_context_len // P) if P else 1
        first = min(shared // P, parts - 1) if P else 0
        if first >= 2:
            per_seq = first * P * w.num_kv_heads * w.head_dim * 2 * w.elem_bytes
            distinct = sb["decode"] - (w.num_seqs - 1) * per_seq
            d_ach = distinct / (att_ms / 1e3) / 1e9
            roof["achieved"] = round(d_ach, 1)
            roof["frac"] = round(d_ach / peak, 4)
            roof["algorithmic_bytes_per_launch"] = int(distinct)
            roof["bytes_note"] = ("distinct K/V bytes: the shared partitions counted once "
                                  f"({first} x {P} tokens), the rest per sequence; "
                                  "kv_gbs counts every sequence's whole context")
            roof["traffic"] = roof["traffic_ratio"] = None
            if ceiling:
                roof["frac_read"] = round(d_ach / ceiling["gbs"], 4)
                roof["frac_read_paged"] = round(d_ach / ceiling["scattered_tiles_gbs"], 4)
    rec = {
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": round(elapsed_ms / K, 5),
        "seq_steps_per_s": round(agg["seqs"] * K / (elapsed_ms / 1e3), 1),
        "hbm_frac_of_peak": round(value / peak, 4),
        "dtype": w.dtype,
        "config": {
            "workload": WORKLOAD_TEXT[name] + (f" [batch overridden to {args.batch}]"
                                               if args.batch is not None and name == args.workload
                                               else ""),
            "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": 16, "partition_tokens": w.partition_tokens,
            "mean_context_len": float(np.mean(w.context_lens)),
            "kv_bytes_per_step": w.kv_bytes(),
            "step": ("copy_blocks + write_kv + attention" if len(w.copy_pairs)
                     else "write_kv + attention") + " (partitions + LSE reduce when split)",
            "scheduler": ("persistent: plan kernel + work-queue grid of SMs x resident CTAs"
                          if res["persistent"] else
                          f"shared prefix: {res['shared_tokens']} shared tokens, their whole "
                          "partitions as one tcgen05 contraction over all sequences, the rest "
                          "as decode partitions" if res.get("shared_tokens") else
                          "longest first, persistent: plan kernel (items in descending key "
                          "count) + one CTA per SM taking (query-tile pair, partition, KV head, "
                          "sequence) items from a work counter" if res.get("tc_path") else
                          "grid: one CTA per (partition, KV head, sequence)"),
            "accumulate": "fp32",
            "l2": l2_note(w),
            "last_block_waste": waste_stats(w),
            "parallelism": f"dp{world} (independent sequences per GPU)",
        },
        "roofline": roof,
        "sub_ms": {"attention": round(att_ms, 5),
                   "write_kv": None if agg["write_ms"] is None else round(agg["write_ms"], 5),
                   "copy_blocks": None if agg["copy_ms"] is None else round(agg["copy_ms"], 5)},
        "op_us": {"write_kv": None if agg["write_ms"] is None else round(agg["write_ms"] * 1e3, 2),
                  "copy_blocks": None if agg["copy_ms"] is None else round(agg["copy_ms"] * 1e3, 2),
                  "copy_blocks_pairs": res["copy_pairs"], "copy_blocks_what": res["copy_what"],
                  "timing": f"each op alone, {res['short_reps']} back-to-back calls queued "
                            f"behind GPU work, events at the loop ends; best of "
                            f"{res['rounds']} loops"},
        "gpu_launches": res["launches"] * K,
        "device_errors": agg["errors"],
    }
    if res["e2e"]:
        e = res["e2e"]
        rec["e2e"] = {"value": round(agg["kv"] * K / (agg["e2e_ms"] / 1e3) / 1e9, 2),
                      "unit": "GB/s", "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                      "ms_per_step": round(agg["e2e_ms"] / K, 5)}
    return rec


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, rank, world)
    if args.op == "blockmgr":
        return run_blockmgr(args) if rank == 0 else 0

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.op == "swap":
        return run_swap(args, device) if rank == 0 else 0
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    names = [args.workload] + [n for n in args.also.split(",") if n and n != args.workload]
    entry_args = {}
    for n in names:
        wl, _, sched = n.partition(":")
        if wl not in WORKLOAD_TEXT or (sched and sched not in ("grid", "persistent", "shared")):
            raise SystemExit(f"unknown workload {n}")
        a = args
        if sched:
            import copy
            a = copy.copy(args)
            a.scheduler = sched
        entry_args[n] = (wl, a)
    records = {}
    ceiling = None
    with ClockSampler(device.index if device.index is not None else 0) as clocks:
        # a buffer 16x the L2: the read-ceiling probe's input, and the GPU work
        # queued ahead of the loops of short calls
        probe_buf = torch.empty(2 << 30, dtype=torch.uint8, device=device)
        if not args.no_read_probe:
            ceiling = read_ceiling(device)
        for i, name in enumerate(names):
            wl, a = entry_args[name]
            res = run_gpu(a, wl, rank, world, device, probe_buf=probe_buf)
            agg = reduce_over_ranks(res, world, device)
            records[name] = (res, agg)
            if i > 0:                  # keep only the headline's pools (the CPU leg reads them)
                res["w"] = _light(res["w"])
            torch.cuda.empty_cache()
        del probe_buf
    head_res, head_agg = records[args.workload]
    rec = workload_record(args.workload, head_res, head_agg, entry_args[args.workload][1], world,
                          ceiling)
    line = {
        "metric": METRIC,
        "value": rec["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": rec["dtype"],
        "data": "synthetic (seeded N(0,1) q/K/V, seeded random block placement)",
    }
    line.update({k: v for k, v in rec.items() if k not in line})
    line["clocks"] = clocks.report()
    if ceiling:
        line["read_ceiling"] = ceiling
    also = {}
    for name in names[1:]:
        wl, a = entry_args[name]
        r = workload_record(wl, *records[name], a, world, ceiling)
        also[name] = r
    if also:
        line["also"] = also
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(head_res["w"], args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(cb["gbs"], 4), "unit": "GB/s", "cores": cb["cores"],
                                "kind": "oracle", "sample": cb["sample"],
                                "seq_steps_per_s": round(cb["seq_steps_per_s"], 3),
                                "seconds": round(cb["seconds"], 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _light(w):
    """A workload without its cache pools (enough for the report)."""
    import dataclasses
    return dataclasses.replace(w, k_pool=w.k_pool[:1], v_pool=w.v_pool[:1])


def main_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands, on the host cores,
    on the same workload, metric and unit. Rank 0 only."""
    if rank != 0:
        return 0
    w = make_workload(args.workload, args.batch)
    vals, secs = [], []
    cb = None
    for _ in range(args.warmup):
        oracle_sample(w, max(0.5, args.cpu_seconds / 10))
    for _ in range(args.steps):
        cb = oracle_sample(w, args.cpu_seconds / max(1, args.steps))
        vals.append(cb["gbs"])
        secs.append(cb["seconds"])
    value = float(np.mean(vals))
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * float(np.mean(secs)), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/K/V, seeded random block placement)",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "num_seqs": w.num_seqs,
                   "partition_tokens": w.partition_tokens,
                   "parallelism": "host threads over (seq, head) rows"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cb["cores"],
                         "kind": "oracle", "sample": cb["sample"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
