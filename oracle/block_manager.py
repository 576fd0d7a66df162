"""Plain-Python model of the host block manager (test infrastructure only).

It states the rules as directly as possible, so that the native manager in
libpa can be compared with it operation by operation:

* "Optimizing LLM Inference: From PagedAttention to AI Infra", "On-Demand
  Allocation": a sequence of n tokens holds ceil(n / 16) blocks; the next
  block is taken only when the last one is full.
* same page, "Copy-on-Write"; "PagedAttention", "KV Cache Sharing
  (Copy-on-Write)": a fork references the same physical blocks; writing into
  a block that other sequences still reference first copies it to a fresh
  block (the last remaining holder writes in place).
* "PagedAttention in Action ...", "Fixed Block Size, Mitigating External
  Fragmentation": blocks nobody references return to the pool.

Free blocks are handed out last-freed first, initially 0, 1, 2, ...; every
operation either completes or leaves the state unchanged (done here by
working on a copy of the state).
"""
from __future__ import annotations

import copy

BLOCK = 16


class OutOfBlocks(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int = BLOCK):
        assert block_size == BLOCK and num_blocks >= 1
        self.num_blocks = num_blocks
        self.ref = [0] * num_blocks
        self.free_list = list(range(num_blocks - 1, -1, -1))   # pop() from the end
        self.seqs: dict[int, dict] = {}                         # id -> {"blocks": [...], "n": tokens}

    # -- helpers
    def _take(self) -> int:
        if not self.free_list:
            raise OutOfBlocks()
        b = self.free_list.pop()
        self.ref[b] = 1
        return b

    def _drop(self, b: int) -> None:
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free_list.append(b)

    def _atomic(self, fn):
        saved = copy.deepcopy((self.ref, self.free_list, self.seqs))
        try:
            return fn()
        except Exception:
            self.ref, self.free_list, self.seqs = saved
            raise

    # -- operations
    def add_sequence(self, sid: int, n: int) -> None:
        if sid in self.seqs or n < 0:
            raise KeyError(sid)

        def run():
            self.seqs[sid] = {"blocks": [self._take() for _ in range(-(-n // BLOCK))], "n": n}
        self._atomic(run)

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.seqs or child in self.seqs or parent == child:
            raise KeyError(child)
        src = self.seqs[parent]
        for b in src["blocks"]:
            self.ref[b] += 1
        self.seqs[child] = {"blocks": list(src["blocks"]), "n": src["n"]}

    def free(self, sid: int) -> None:
        for b in self.seqs.pop(sid)["blocks"]:
            self._drop(b)

    def slot(self, sid: int, pos: int) -> int:
        s = self.seqs[sid]
        assert 0 <= pos < s["n"]
        return s["blocks"][pos // BLOCK] * BLOCK + pos % BLOCK

    def append_slots(self, ids):
        if len(set(ids)) != len(ids) or any(i not in self.seqs for i in ids):
            raise KeyError(ids)

        def run():
            slots, cow = [], []
            for sid in ids:
                s = self.seqs[sid]
                pos = s["n"]
                if pos % BLOCK == 0:                 # last block full (or none): a new one
                    s["blocks"].append(self._take())
                elif self.ref[s["blocks"][-1]] > 1:  # shared: copy before writing
                    old = s["blocks"][-1]
                    new = self._take()
                    self._drop(old)
                    s["blocks"][-1] = new
                    cow.append((old, new))
                slots.append(s["blocks"][-1] * BLOCK + pos % BLOCK)
                s["n"] = pos + 1
            return slots, cow
        return self._atomic(run)

    def block_tables(self, ids, stride: int):
        rows, lens = [], []
        for sid in ids:
            s = self.seqs[sid]
            if len(s["blocks"]) > stride:
                raise ValueError("stride")
            rows.append(s["blocks"] + [-1] * (stride - len(s["blocks"])))
            lens.append(s["n"])
        return rows, lens

    def stats(self) -> dict:
        used = self.num_blocks - len(self.free_list)
        return {"num_blocks": self.num_blocks, "free_blocks": len(self.free_list),
                "used_blocks": used, "shared_blocks": sum(r > 1 for r in self.ref),
                "sequences": len(self.seqs), "tokens": sum(s["n"] for s in self.seqs.values()),
                "logical_blocks": sum(len(s["blocks"]) for s in self.seqs.values())}
