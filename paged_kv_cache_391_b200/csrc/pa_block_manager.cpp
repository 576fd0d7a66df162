// pa_block_manager.cpp -- host-side block manager for the paged KV cache.
//
// What it follows:
//  * "Optimizing LLM Inference: From PagedAttention to AI Infra", "On-Demand
//    Allocation": a sequence holds only the blocks its tokens fill; a new
//    block is taken when the last one is full (35 tokens -> 3 blocks).
//  * same page, "Copy-on-Write", and "PagedAttention", "KV Cache Sharing
//    (Copy-on-Write)": forked sequences reference the same physical blocks;
//    a block is copied only when a sequence writes into a block others still
//    hold, and the shared original stays unchanged.
//  * "PagedAttention in Action ...", "Fixed Block Size, Mitigating External
//    Fragmentation": released blocks return to one pool of same-sized blocks.
//  * "The Memory Wall ...", "The Block Manager": the scheduler asks the block
//    manager whether enough free blocks remain.
//
// Data structures: a reference count per physical block, a LIFO stack of free
// block ids (initially 0, 1, 2, ... from the top), and per sequence its list
// of physical blocks and token count. Every operation either succeeds
// completely or changes nothing. Not thread-safe: one manager per scheduler.
#include <stdint.h>

#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pa.h"

struct pa_block_manager {
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t num_tokens = 0;
  };
  int64_t num_blocks = 0;
  std::vector<int32_t> refcount;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::unordered_map<int64_t, Seq> seqs;

  int32_t pop() {
    const int32_t b = free_stack.back();
    free_stack.pop_back();
    refcount[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--refcount[b] == 0) free_stack.push_back(b);
  }
};

namespace {
constexpr int64_t kBlock = PA_BLOCK_SIZE;
int64_t blocks_for(int64_t tokens) { return (tokens + kBlock - 1) / kBlock; }
}  // namespace

extern "C" {

pa_block_manager* pa_bm_create(int64_t num_blocks, int32_t block_size) {
  if (num_blocks < 1 || num_blocks > INT32_MAX || block_size != PA_BLOCK_SIZE) return nullptr;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (!bm) return nullptr;
  try {
    bm->num_blocks = num_blocks;
    bm->refcount.assign((size_t)num_blocks, 0);
    bm->free_stack.reserve((size_t)num_blocks);
    for (int64_t b = num_blocks - 1; b >= 0; --b) bm->free_stack.push_back((int32_t)b);
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int64_t pa_bm_num_free_blocks(const pa_block_manager* bm) {
  return bm ? (int64_t)bm->free_stack.size() : -1;
}

pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int64_t num_tokens) {
  if (!bm || num_tokens < 0 || bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  const int64_t n = blocks_for(num_tokens);
  if (n > (int64_t)bm->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq s;
  s.num_tokens = num_tokens;
  s.blocks.reserve((size_t)n);
  for (int64_t i = 0; i < n; ++i) s.blocks.push_back(bm->pop());
  bm->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
  if (!bm || parent_id == child_id || bm->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  pa_block_manager::Seq child = it->second;
  for (int32_t b : child.blocks) ++bm->refcount[b];
  bm->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  for (int32_t b : it->second.blocks) bm->release(b);
  bm->seqs.erase(it);
  return PA_OK;
}

pa_status pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int64_t start, int64_t count,
                      int64_t* slots) {
  if (!bm || start < 0 || count < 0 || (count > 0 && !slots)) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || start + count > it->second.num_tokens) return PA_ERR_INVALID_ARG;
  for (int64_t t = 0; t < count; ++t) {
    const int64_t pos = start + t;
    slots[t] = (int64_t)it->second.blocks[(size_t)(pos / kBlock)] * kBlock + pos % kBlock;
  }
  return PA_OK;
}

pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                             int64_t* slot_mapping, int64_t* cow_pairs, int32_t* num_cow) {
  if (!bm || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !slot_mapping || !cow_pairs)) ||
      !num_cow)
    return PA_ERR_INVALID_ARG;
  // Pass 1: validate and count the blocks this step takes, replaying the
  // reference-count changes in order (a shared last block is copied by every
  // writer but the last one still holding it), without changing anything.
  std::vector<pa_block_manager::Seq*> seq_ptrs((size_t)num_seqs);
  std::unordered_set<int64_t> seen;
  std::unordered_map<int32_t, int32_t> released;  // block -> references dropped in this step
  int64_t need = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || !seen.insert(seq_ids[i]).second) return PA_ERR_INVALID_ARG;
    pa_block_manager::Seq& s = it->second;
    seq_ptrs[(size_t)i] = &s;
    if (s.num_tokens % kBlock == 0) {
      ++need;  // the last block is full (or there is none): take a new one
    } else {
      const int32_t last = s.blocks.back();
      const int32_t refs = bm->refcount[last] - released[last];
      if (refs > 1) {
        ++need;  // copy-on-write
        ++released[last];
      }
    }
  }
  if (need > (int64_t)bm->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
  // Pass 2: apply.
  int32_t nc = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    pa_block_manager::Seq& s = *seq_ptrs[(size_t)i];
    const int64_t off = s.num_tokens % kBlock;
    int32_t blk;
    if (off == 0) {
      blk = bm->pop();
      s.blocks.push_back(blk);
    } else {
      blk = s.blocks.back();
      if (bm->refcount[blk] > 1) {
        const int32_t fresh = bm->pop();
        bm->release(blk);
        cow_pairs[2 * nc] = blk;
        cow_pairs[2 * nc + 1] = fresh;
        ++nc;
        s.blocks.back() = fresh;
        blk = fresh;
      }
    }
    slot_mapping[i] = (int64_t)blk * kBlock + off;
    ++s.num_tokens;
  }
  *num_cow = nc;
  return PA_OK;
}

pa_status pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids,
                             int32_t num_seqs, int32_t* block_tables, int32_t stride,
                             int32_t* context_lens) {
  if (!bm || num_seqs < 0 || stride < 1 ||
      (num_seqs > 0 && (!seq_ids || !block_tables || !context_lens)))
    return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < num_seqs; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
    if ((int64_t)it->second.blocks.size() > stride || it->second.num_tokens > INT32_MAX)
      return PA_ERR_INVALID_ARG;
  }
  for (int32_t i = 0; i < num_seqs; ++i) {
    const pa_block_manager::Seq& s = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = block_tables + (size_t)i * stride;
    const size_t n = s.blocks.size();
    for (size_t j = 0; j < (size_t)stride; ++j) row[j] = j < n ? s.blocks[j] : -1;
    context_lens[i] = (int32_t)s.num_tokens;
  }
  return PA_OK;
}

pa_status pa_bm_get_stats(const pa_block_manager* bm, pa_bm_stats* out) {
  if (!bm || !out) return PA_ERR_INVALID_ARG;
  pa_bm_stats st{};
  st.num_blocks = bm->num_blocks;
  st.free_blocks = (int64_t)bm->free_stack.size();
  st.used_blocks = st.num_blocks - st.free_blocks;
  for (int32_t r : bm->refcount) st.shared_blocks += r > 1;
  st.sequences = (int64_t)bm->seqs.size();
  for (const auto& kv : bm->seqs) {
    st.tokens += kv.second.num_tokens;
    st.logical_blocks += (int64_t)kv.second.blocks.size();
  }
  *out = st;
  return PA_OK;
}

int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->refcount[(size_t)block];
}

}  // extern "C"
