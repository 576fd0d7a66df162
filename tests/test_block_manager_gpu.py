"""The block manager driving the kernels: several decode steps with prompts,
forks (copy-on-write on the first divergent token), a freed sequence whose
blocks are reused, and new arrivals. Each step's slot mapping, copy pairs,
tables and lengths come from the native manager; libpa's kernels and the
oracle both consume them; pools must match bit for bit and outputs within
the decode tolerance, at every step."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_391_b200 import pa
from paged_kv_cache_391_b200 import workloads as W

from gpu_helpers import assert_decode_close, dev16, host16, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hq,Hkv,D,dtype", [(8, 2, 128, "bf16"), (4, 4, 64, "f16")])
def test_block_manager_drives_decode_steps(Hq, Hkv, D, dtype):
    rng = np.random.default_rng(31 + Hq)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    NB, stride = 400, 64
    bm = pa.BlockManager(NB)
    nan = W.NAN_BITS[dtype]
    kp = np.full((NB, Hkv, 16, D), nan, np.uint16)
    vp = kp.copy()
    kc, vc = dev16(kp, tdt), dev16(vp, tdt)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def prefill(sid, n):
        bm.add_sequence(sid, n)
        k = W._normal_bits(rng, (n, Hkv, D), dtype)
        v = W._normal_bits(rng, (n, Hkv, D), dtype)
        slots = bm.slots(sid, 0, n)
        oracle.write_kv(k, v, kp, vp, slots)
        pa.write_kv(dev16(k, tdt), dev16(v, tdt), kc, vc, torch.from_numpy(slots).cuda(),
                    dev_error=err)

    prefill(0, 37)
    prefill(1, 100)
    prefill(2, 16)
    bm.fork(1, 3)                     # two samples of one prompt
    bm.fork(1, 4)
    live = [0, 1, 2, 3, 4]
    n_cow = 0
    for step in range(12):
        if step == 4:
            bm.free(2)
            live.remove(2)            # its blocks go back to the pool ...
        if step == 5:
            prefill(5, 70)            # ... and a new arrival takes them
            live.append(5)
        if step == 8:
            bm.fork(5, 6)
            live.append(6)
        slots, cow = bm.append_slots(live)
        n_cow += len(cow)
        S = len(live)
        new_k = W._normal_bits(rng, (S, Hkv, D), dtype)
        new_v = W._normal_bits(rng, (S, Hkv, D), dtype)
        q = W._normal_bits(rng, (S, Hq, D), dtype)
        bt, lens = bm.block_tables(live, stride)
        if len(cow):
            oracle.copy_blocks([kp], [vp], cow)
            pa.copy_blocks([kc], [vc], torch.from_numpy(cow).cuda(), dev_error=err)
        oracle.write_kv(new_k, new_v, kp, vp, slots)
        pa.write_kv(dev16(new_k, tdt), dev16(new_v, tdt), kc, vc, torch.from_numpy(slots).cuda(),
                    dev_error=err)
        out = torch.empty((S, Hq, D), dtype=tdt, device="cuda")
        pa.decode(out, dev16(q, tdt), kc, vc, torch.from_numpy(bt).cuda(),
                  torch.from_numpy(lens).cuda(), scale=1 / np.sqrt(D),
                  max_context_len=int(lens.max()), partition_tokens=32, dev_error=err)
        torch.cuda.synchronize()
        assert np.array_equal(host16(kc), kp) and np.array_equal(host16(vc), vp), step
        ref = oracle.decode(q, kp, vp, bt, lens, 1 / np.sqrt(D), dtype)
        assert_decode_close(to_f64(out), ref, f"step {step}")
    assert int(err.item()) == 0
    assert n_cow == 2 + 1             # forks of seq 1 (two copies), fork of seq 5 (one)
