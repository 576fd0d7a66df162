// pa_prefill_tc.cu -- chunked-prefill attention over the paged cache on the
// fifth-generation tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes is pa_prefill_chunk: the last Tq tokens of a sequence's
// context are queries, query token t attends to context positions
// 0 .. L - Tq + t ("PagedAttention in Action ...", "Chunked Prefill"; the
// block table walk of "PagedAttention: Decoupling Logical Context ...").
// With many query rows per KV head this is a dense contraction, so it runs on
// tcgen05 instead of the 16-row mma.sync tiles of the decode kernel.
//
// A work item is a (pair of 128-row query tiles, partition, KV head,
// sequence); tile rows are (query token, head) pairs of the KV head's query
// group. Both tiles share every K/V tile loaded for the item. Without a plan
// one CTA runs one item (grid order); with the plan (longest first) one CTA
// per SM runs items from a work counter until the list is exhausted, keeping
// its TMEM, barriers and rings across items. 320 threads, one CTA per SM:
//  * warps 0-3 and 4-7: softmax of tile 0 and tile 1. Thread r of a
//    warpgroup owns row r of its tile: TMEM lane r of its S, P and O.
//  * warp 8: TMA loads (per step K and V of 8 cache blocks = 128 keys, each in
//    its own 2-stage ring, sixteen lanes issuing a ring's sixteen boxes; an
//    item's Q after its first K and V) and, with the plan, the next item.
//  * warp 9, one lane: every MMA:
//      S_i(j)  = Q_i K_j^T      (M=128, N=128 keys, K=D; Q, K K-major in smem)
//      O_i    += P_i(j) V_j     (M=128, N=D, K=128 keys; P in TMEM, V MN-major
//                                in smem)
//    P_i(j) (bf16) is written by the softmax over the first 64 columns of
//    S_i(j), so the tensor core reads only V from shared memory for P.V and
//    Q, K for S: per 128 keys 8 KiB of operands per 64-cycle MMA at most.
//    Issue order S_0(j), P.V_1(j-1), S_1(j), P.V_0(j), S_0(j+1), ...: each
//    tile's softmax has the time of two MMA groups (the other tile's) to
//    finish, the two softmaxes alternate instead of competing, and S_i(j+1)
//    is issued after P.V_i(j), which has read P_i(j) from the same columns
//    (tcgen05 MMAs of one thread run in issue order). The commit that
//    signals S_i(j) also covers P.V_i(j-1), so the softmax may rescale O_i
//    as soon as it sees S_i(j).
//    TMEM: tile i at columns 256 i: S (P over its first half) [0,128),
//    O [128,256).
// Online softmax per row in fp32, base 2 (hardware ex2); a row's reference
// maximum and O are only rescaled when the maximum grows by more than 2^8.
// Keys past the context, past the row's causal limit, or in a block with a bad
// table entry are masked to -inf, and V rows past the context are zeroed
// before P.V (0 * stale data must stay 0). All waits are bounded; TMEM is
// released on every path.
#include <math.h>

#include <type_traits>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;                 // query rows per tile (M)
constexpr int kTiles = 2;                  // query tiles per CTA
constexpr int kKeys = 128;                 // keys per step (8 cache blocks)
constexpr int kStepBlocks = kKeys / 16;
constexpr int kD = 128;                    // head dim of this path
constexpr int kChunks = kD / 64;           // 128-byte swizzle columns of a row
constexpr int kStages = 2;                 // K and V ring depth
constexpr int kSoftmaxWarps = 4 * kTiles;
constexpr int kLoadWarp = kSoftmaxWarps;       // TMA loads
constexpr int kMmaWarp = kSoftmaxWarps + 1;    // tcgen05.mma issue
constexpr int kThreadsTc = (kSoftmaxWarps + 2) * 32;
constexpr uint32_t kTileCols = 256;        // per tile: S / P [0,128), O [128,256)
constexpr uint32_t kTmemCols = kTiles * kTileCols;
constexpr uint32_t kOCol = 128;

constexpr int kQBytes = kRows * kD * 2;            // 32 KiB per tile: [chunk][128 rows][128 B]
constexpr int kKBytes = kKeys * kD * 2;            // 32 KiB: [chunk][128 keys][128 B]
constexpr int kVBytes = kKeys * kD * 2;            // 32 KiB: [chunk][128 keys][128 B]
constexpr int kQOff = 0;                           // Q tiles 0, 1
constexpr int kKOff = kTiles * kQBytes;            // K stages
constexpr int kVOff = kKOff + kStages * kKBytes;   // V stages
constexpr int kBarOff = kVOff + kStages * kVBytes;
// barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2],
// s_full[2 tiles], p_ready[2 tiles], o_done, mma_drain, q_empty,
// item_full[2], item_empty[2]; then the two item slots and the TMEM address
constexpr int kNumBars = 1 + 4 * kStages + 2 * kTiles + 2 + 1 + 4;
constexpr int kItemSlotOff = kBarOff + kNumBars * 8;
constexpr int kTmemSlotOff = kItemSlotOff + 8;
constexpr int kSmemBytes = kTmemSlotOff + 16;
// The dynamic shared memory is declared 1024-byte aligned and the kernel
// checks it (no slack is reserved).
constexpr int kSmemAlloc = kSmemBytes;
static_assert(kSmemAlloc <= 227 * 1024, "one CTA per SM must fit");

// 2^x by the hardware approximation (ex2.approx, relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input max / min (one instruction on sm_100): the softmax is bound by
// instruction issue, and its row-maximum reduction halves with them.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// A row's running maximum is only moved (and O rescaled) when the new
// maximum exceeds it by more than 2^8: until then P is taken against the
// older, smaller reference (values up to 256, exact in the fp32 sums and
// representable in bf16), and O / l is unchanged by the choice of reference.
constexpr float kRescaleLog2 = 8.f;

// One unit of the chunk kernel's work: a pair of query tiles of one
// sequence's chunk, one partition of its keys, one KV head; and what every
// role derives from it (uniform over the CTA).
struct ChunkItem {
  int seq, kvh, part, qtile;  // qtile: the pair's first tile
  int L, q0, Tq, t0, n_parts, key_begin, key_end, n_steps;
  bool skip;                  // no rows or no keys of this item exist
  bool causal;                // query token t sees keys up to L - Tq + t (else all L)
  int err_count;              // argument errors this item counts (its first item only)
};

__device__ __forceinline__ ChunkItem chunk_item(int seq, int kvh, int part, int qtile,
                                                const int32_t* __restrict__ q_start,
                                                int num_q_tokens, int max_query_len,
                                                const int32_t* __restrict__ context_lens,
                                                int group, int max_context_len, int part_blocks,
                                                int shared_L) {
  ChunkItem it;
  it.seq = seq;
  it.kvh = kvh;
  it.part = part;
  it.qtile = qtile;
  it.err_count = 0;
  it.skip = false;
  it.causal = shared_L < 0;
  if (shared_L >= 0) {
    // A shared prefix: every row of q (one query token per sequence) sees
    // all shared_L keys of sequence 0's table (checked by the host and the
    // decode kernel), no mask.
    const int tok_per_tile = kRows / group;
    it.seq = 0;
    it.L = shared_L;
    it.q0 = 0;
    it.Tq = num_q_tokens;
    it.t0 = qtile * tok_per_tile;
    const int nblk = (shared_L + 15) / 16;
    it.n_parts = nblk > 0 ? (nblk + part_blocks - 1) / part_blocks : 1;
    it.key_begin = part * part_blocks * 16;
    it.key_end = min((part + 1) * part_blocks * 16, shared_L);
    it.skip = it.t0 >= it.Tq || part >= it.n_parts;
    it.n_steps = !it.skip && it.key_end > it.key_begin
                     ? (it.key_end - it.key_begin + kKeys - 1) / kKeys : 0;
    return it;
  }
  const bool counts = part == 0 && kvh == 0 && qtile == 0;
  int L = context_lens[seq];
  if (L < 0 || L > max_context_len) {
    it.err_count += counts;
    L = L < 0 ? 0 : max_context_len;
  }
  it.L = L;
  it.q0 = q_start[seq];
  int Tq = q_start[seq + 1] - it.q0;
  it.n_steps = 0;
  it.t0 = 0;
  it.n_parts = 1;
  it.key_begin = it.key_end = 0;
  if (it.q0 < 0 || Tq < 0 || it.q0 + Tq > num_q_tokens) {
    it.err_count += counts;
    it.Tq = 0;
    it.skip = true;
    return it;
  }
  if (Tq > min(L, max_query_len)) {
    it.err_count += counts;
    Tq = min(L, max_query_len);
  }
  it.Tq = Tq;
  const int tok_per_tile = kRows / group;
  it.t0 = qtile * tok_per_tile;
  const int nblk_seq = (L + 15) / 16;
  it.n_parts = nblk_seq > 0 ? (nblk_seq + part_blocks - 1) / part_blocks : 1;
  if (it.t0 >= Tq || part >= it.n_parts) {
    it.skip = true;
    return it;
  }
  it.key_begin = part * part_blocks * 16;
  const int t_last = min(it.t0 + kTiles * tok_per_tile, Tq) - 1;  // the pair's last query token
  // keys the pair can see in this partition: up to the last row's causal limit
  it.key_end = min(min((part + 1) * part_blocks * 16, L), L - Tq + t_last + 1);
  it.n_steps = it.key_end > it.key_begin ? (it.key_end - it.key_begin + kKeys - 1) / kKeys : 0;
  return it;
}

// Grid mode runs the one item its block index names. Plan mode is persistent:
// one CTA per SM, each taking items of the plan's list (longest first) from a
// work counter until the list is exhausted. The TMA warp takes the next item
// once it has issued every load of the current one and posts it in a
// two-slot ring (item_full / item_empty) for the MMA and softmax warps; so the
// next item's Q and first K / V loads overlap the current item's end, and the
// TMEM allocation, the barriers and their phases carry over between items.
template <typename T>
__global__ void __launch_bounds__(kThreadsTc, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, T* __restrict__ out,
                      float* __restrict__ part_o, float* __restrict__ part_lse,
                      const int32_t* __restrict__ q_start, int num_q_tokens, int max_query_len,
                      const int32_t* __restrict__ block_tables, int bt_stride,
                      const int32_t* __restrict__ context_lens, int num_q_heads, int group,
                      int64_t num_blocks, int max_context_len, float scale_log2,
                      int part_blocks, int max_parts, int32_t* __restrict__ dev_error,
                      const uint2* __restrict__ items, int32_t* __restrict__ plan,
                      int num_kv_heads, int shared_L) {
  using E = Elem<T>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                      // [stage]
  uint64_t* k_empty = k_full + kStages;             // [stage]
  uint64_t* v_full = k_empty + kStages;             // [stage]
  uint64_t* v_empty = v_full + kStages;             // [stage]
  uint64_t* s_full = v_empty + kStages;             // [tile]
  uint64_t* p_ready = s_full + kTiles;              // [tile]
  uint64_t* o_done = p_ready + kTiles;              // an item's O final
  uint64_t* mma_drain = o_done + 1;                 // failure path only
  uint64_t* q_empty = mma_drain + 1;                // an item's last S MMAs done: Q reusable
  uint64_t* item_full = q_empty + 1;                // [2] plan mode: an item posted
  uint64_t* item_empty = item_full + 2;             // [2] plan mode: an item read by all roles
  int32_t* item_slot = reinterpret_cast<int32_t*>(smem + kItemSlotOff);  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemSlotOff);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (smem_addr(smem) & 1023) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && dev_error)
      atomicAdd(dev_error, 1);
    return;
  }
  // The item with index w into the plan's list x KV heads, or (kGridItem) the
  // one the block index names. Recomputed where needed rather than kept.
  constexpr int kGridItem = -2;
  auto item_of = [&](int w) {
    int seq, kvh, part, qtile;
    if (w == kGridItem) {
      seq = blockIdx.z;
      kvh = blockIdx.y;
      part = (int)(blockIdx.x % (unsigned)max_parts);
      qtile = (int)(blockIdx.x / (unsigned)max_parts) * kTiles;
    } else {
      const uint2 pi = items[w / num_kv_heads];
      seq = (int)pi.x;
      kvh = w % num_kv_heads;
      part = (int)(pi.y % (unsigned)max_parts);
      qtile = (int)(pi.y / (unsigned)max_parts) * kTiles;
    }
    return chunk_item(seq, kvh, part, qtile, q_start, num_q_tokens, max_query_len,
                      context_lens, group, max_context_len, part_blocks, shared_L);
  };
  const bool persistent = plan != nullptr;
  if (persistent) {
    griddep_wait();  // the plan kernel's list and zeroed counter are complete and visible
  } else {
    const ChunkItem it = item_of(kGridItem);
    if (tid == 0 && it.err_count && dev_error) atomicAdd(dev_error, it.err_count);
    if (it.skip) {  // uniform over the CTA, before any barrier
      if (shared_L >= 0) griddep_wait();  // see the end of the kernel
      return;
    }
  }

  // ---- set-up: barriers (thread 0), TMEM (warp 0)
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kTiles; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 4 * 32);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_drain, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 1 + kSoftmaxWarps);  // the MMA warp, each softmax warp
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  // The k-th item of this CTA, for the MMA and softmax warps (whole warp): its
  // index into the plan's list x KV heads, kGridItem in grid mode, or -1 when
  // there is none (or the wait for it gave up: failed is then set).
  auto take_item = [&](int k) -> int {
    if (!persistent) return k == 0 ? kGridItem : -1;
    const int slot = k & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&item_full[slot], (uint32_t)((k >> 1) & 1)))) {
      failed = true;
      return -1;
    }
    const int w = *reinterpret_cast<volatile int32_t*>(&item_slot[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[slot]);
    return w;
  };

  const uint32_t q_s = smem_addr(smem + kQOff);
  auto stage_k = [&](int st) { return smem + kKOff + st * kKBytes; };
  auto stage_v = [&](int st) { return smem + kVOff + st * kVBytes; };

  if (warp == kLoadWarp) {
    // ============================ TMA loads =================================
    // The whole warp runs the control flow, so the block table is read 32
    // entries per coalesced load and broadcast by shuffle. Per step and ring
    // (K, then V) lane 0 posts the expected bytes and lanes 0-15 issue the
    // step's sixteen box copies (8 cache blocks x 2 column chunks) in one
    // instruction. A stage is refilled once the MMAs that read it committed
    // its "empty" barrier; the loads run up to kStages steps ahead, across
    // items. An item's Q follows its first K and V, once the previous item's
    // last S MMAs are done with the Q tiles.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int nk = 0, nv = 0, nq = 0;  // K / V steps and Q loads issued, over all items
    // plan mode: the next item, fetched by lane 0 and posted in its slot
    auto fetch_item = [&](int k) {
      const int slot = k & 1;
      if (k >= 2 && !wait_all(&item_empty[slot], (uint32_t)(((k >> 1) - 1) & 1))) {
        failed = true;
        return -1;
      }
      int w = -1;
      if (lane == 0) {
        const int64_t n_work = (int64_t)plan[0] * num_kv_heads;
        const int64_t c = atomicAdd(&plan[1], 1);
        w = c < n_work ? (int)c : -1;
        item_slot[slot] = w;
        mbar_arrive(&item_full[slot]);  // release: the slot write is visible to its waiters
      }
      return __shfl_sync(0xffffffffu, w, 0);
    };
    for (int k = 0; !failed; ++k) {
      const int w = persistent ? fetch_item(k) : (k == 0 ? kGridItem : -1);
      if (w == -1) break;
      const ChunkItem it = item_of(w);
      if (it.skip || it.n_steps == 0) continue;
      const int32_t* bt_row = block_tables + (size_t)it.seq * bt_stride;
      const int lb_first = it.key_begin / 16;
      const int nblk_keys = (it.key_end - it.key_begin + 15) / 16;
      const int tok_per_tile = kRows / group;
      // A table entry outside the pool is skipped (not loaded; the softmax
      // masks its keys) and counted once: by the KV-head-0 item of the last
      // pair of query tiles, whose causal horizon covers the whole partition.
      const bool count_bad = dev_error && it.kvh == 0 && it.t0 + kTiles * tok_per_tile >= it.Tq;
      auto load_window = [&](int wi) {  // entries 32 wi .. 32 wi + 31 of the item's keys
        const int i = 32 * wi + lane;
        int p = -1;
        if (i < nblk_keys) {
          p = __ldg(bt_row + lb_first + i);
          if (p < 0 || p >= num_blocks) {
            if (count_bad) atomicAdd(dev_error, 1);
            p = -1;
          }
        }
        return p;
      };
      int win = 0, pid_cur = load_window(0), pid_nxt = load_window(1);
      auto pid_of = [&](int i) {  // all lanes; i / 32 uniform over the warp
        const int wi = i >> 5;
        if (wi != win && wi != win + 1) {  // outside the register window: read the table
          const int p = i < nblk_keys ? __ldg(bt_row + lb_first + i) : -1;
          return (p < 0 || p >= num_blocks) ? -1 : p;
        }
        const int v = wi == win ? pid_cur : pid_nxt;
        return __shfl_sync(0xffffffffu, v, i & 31);
      };
      // K (or V) of the item's step j (global step g) into stage g % kStages;
      // blocks past the keys or with a bad table entry are not loaded.
      auto load = [&](int j, int g, bool is_v) {
        const int st = g % kStages;
        uint64_t* bar = is_v ? &v_full[st] : &k_full[st];
        uint8_t* dst = is_v ? stage_v(st) : stage_k(st);
        const CUtensorMap* map = is_v ? &tm_v : &tm_k;
        while (((j * kStepBlocks) >> 5) > win) {  // a step's 8 entries share one window
          ++win;
          pid_cur = pid_nxt;
          pid_nxt = load_window(win + 1);
        }
        const int b = (lane >> 1) & (kStepBlocks - 1), c = lane & 1;  // lanes 0-15: block, chunk
        const int pid = pid_of(j * kStepBlocks + b);
        const bool mine = lane < kStepBlocks * kChunks && pid >= 0;
        const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xffffffffu, mine)) * 2048u;
        if (lane == 0) {
          if (bytes) mbar_arrive_expect_tx(bar, bytes);
          else mbar_arrive(bar);  // nothing to load: complete the phase empty
        }
        __syncwarp();
        if (mine) tma_load_4d(dst + c * (kKeys * 128) + b * 2048, map, bar, c * 64, 0, it.kvh, pid);
      };
      for (int j = 0; j < it.n_steps; ++j) {
        if (nk >= kStages &&
            !wait_all(&k_empty[nk % kStages], (uint32_t)((nk / kStages - 1) & 1))) { failed = true; break; }
        load(j, nk, false);
        ++nk;
        if (nv >= kStages &&
            !wait_all(&v_empty[nv % kStages], (uint32_t)((nv / kStages - 1) & 1))) { failed = true; break; }
        load(j, nv, true);
        ++nv;
        if (j == 0) {
          // Q of both tiles (rows past the q buffer read as zeros and are
          // never written out), once the previous item's S MMAs are done
          if (nq > 0 && !wait_all(q_empty, (uint32_t)((nq - 1) & 1))) { failed = true; break; }
          if (lane == 0) {
            if (nq == 0) tma_prefetch_desc(&tm_q);
            mbar_arrive_expect_tx(q_full, kTiles * kQBytes);
#pragma unroll
            for (int i = 0; i < kTiles; ++i)
#pragma unroll
              for (int c = 0; c < kChunks; ++c)
                tc::tma_load_3d(smem + kQOff + i * kQBytes + c * (kRows * 128), &tm_q, q_full,
                                c * 64, it.kvh * group, it.q0 + it.t0 + i * tok_per_tile);
          }
          ++nq;
        }
      }
    }
    if (failed) {
      // Let the copies already issued land (each wait bounded) before the
      // shared memory is released.
      if (nq > 0) (void)mbar_wait(q_full, (uint32_t)((nq - 1) & 1));
      for (int st = 0; st < kStages; ++st) {
        // the last load issued into stage st is number st + kStages * ((n - 1 - st) / kStages)
        if (nk > st) (void)mbar_wait(&k_full[st], (uint32_t)(((nk - 1 - st) / kStages) & 1));
        if (nv > st) (void)mbar_wait(&v_full[st], (uint32_t)(((nv - 1 - st) / kStages) & 1));
      }
      if (lane == 0 && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
    }
  } else if (warp == kMmaWarp) {
    // ============================== MMAs ====================================
    // One lane issues every tcgen05.mma in the order S_0(j), P.V_1(j-1),
    // S_1(j), P.V_0(j) within an item, then the item's last P.V_1; the next
    // item's S_0(0) follows at once. Descriptors are built once and offset
    // per MMA; g counts steps over all items (ring stages and barrier phases).
    const bool leader = lane == 0;
    const uint32_t id_s = tc::instr_desc_f16(Elem<T>::kBf16, kRows, kKeys, false, false);
    const uint32_t id_pv = tc::instr_desc_f16(Elem<T>::kBf16, kRows, kD, false, true);
    const uint64_t dq = tc::smem_desc_sw128(q_s, 16, 1024);
    const uint64_t dk = tc::smem_desc_sw128(smem_addr(stage_k(0)), 16, 1024);
    const uint64_t dv = tc::smem_desc_sw128(smem_addr(stage_v(0)), kKeys * 128, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    // S_i = Q_i K^T of global step g into tile i's S columns; commit to s_full[i]
    auto issue_s = [&](int i, int g) {
      const uint64_t dks = dk + (uint64_t)(((g % kStages) * kKBytes) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 columns = 32 bytes into the row
          const uint64_t a = dq + (uint64_t)((i * kQBytes + (kk >> 2) * (kRows * 128) + off) >> 4);
          const uint64_t b = dks + (uint64_t)(((kk >> 2) * (kKeys * 128) + off) >> 4);
          tc::mma_f16(tmem + (uint32_t)(i * kTileCols), a, b, id_s, kk > 0);
        }
        tc::commit(&s_full[i]);
      }
    };
    // O_i += P_i V of global step g, P from TMEM (the first 64 columns of tile
    // i's S); `first`: the item's first step (O starts from zero)
    auto issue_pv = [&](int i, int g, bool first) {
      const uint64_t dvs = dv + (uint64_t)(((g % kStages) * kVBytes) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t b = dvs + (uint64_t)((kk * 2048) >> 4);
          tc::mma_f16_tmem_a(tmem + (uint32_t)(i * kTileCols) + kOCol,
                             tmem + (uint32_t)(i * kTileCols) + (uint32_t)(kk * 8), b, id_pv,
                             !first || kk > 0);
        }
      }
    };
    int g0 = 0, nq = 0;  // steps and Q tiles consumed by earlier items
    for (int k = 0; !failed; ++k) {
      const int w = take_item(k);
      if (w == -1) break;
      const ChunkItem it = item_of(w);
      if (it.skip || it.n_steps == 0) continue;
      const int n = it.n_steps;
      if (!wait_all(q_full, (uint32_t)(nq & 1))) { failed = true; break; }
      ++nq;
      for (int j = 0; j < n; ++j) {
        const int g = g0 + j, st = g % kStages;
        if (!wait_all(&k_full[st], (uint32_t)((g / kStages) & 1))) { failed = true; break; }
        tc::fence_after_sync();
        issue_s(0, g);
        if (j > 0) {  // P.V_1(j-1): V(j-1) landed (awaited before P.V_0(j-1))
          if (!wait_all(&p_ready[1], (uint32_t)((g - 1) & 1))) { failed = true; break; }
          tc::fence_after_sync();
          issue_pv(1, g - 1, j == 1);
          if (leader) tc::commit(&v_empty[(g - 1) % kStages]);
        }
        issue_s(1, g);
        if (leader) {
          tc::commit(&k_empty[st]);  // K stage st free once S_0, S_1 of step g completed
          if (j == n - 1) tc::commit(q_empty);  // the item's last S MMAs: Q reusable after them
        }
        if (!wait_all(&v_full[st], (uint32_t)((g / kStages) & 1))) { failed = true; break; }
        if (!wait_all(&p_ready[0], (uint32_t)(g & 1))) { failed = true; break; }
        tc::fence_after_sync();
        issue_pv(0, g, j == 0);
      }
      if (failed) break;
      const int gl = g0 + n - 1;
      if (!wait_all(&p_ready[1], (uint32_t)(gl & 1))) { failed = true; break; }
      tc::fence_after_sync();
      issue_pv(1, gl, n == 1);
      if (leader) {
        tc::commit(&v_empty[gl % kStages]);
        tc::commit(o_done);  // both tiles' O of the item are final once this completes
      }
      g0 += n;
    }
    if (failed) {
      // The MMAs already issued finish (bounded wait) before TMEM is released:
      // a commit covers every MMA this thread issued before it. o_done stays
      // unsignalled, so the softmax warps time out instead of reading O.
      if (leader) tc::commit(mma_drain);
      (void)mbar_wait(mma_drain, 0);
      if (leader && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
    }
  } else {
    // =============================== softmax ================================
    const int tile = warp >> 2;                          // this warpgroup's query tile
    const int r = tid & (kRows - 1);                     // tile row = TMEM lane
    const uint32_t lane_addr =
        tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(tile * kTileCols);
    int g = 0, no = 0;  // steps (over all items) and O results consumed so far
    for (int k = 0; !failed; ++k) {
      const int w = take_item(k);
      if (w == -1) break;
      const ChunkItem it = item_of(w);
      if (persistent && tid == 0 && it.err_count && dev_error) atomicAdd(dev_error, it.err_count);
      if (it.skip) continue;
      const int key_begin = it.key_begin, key_end = it.key_end, seq = it.seq;
      const int L = it.L, Tq = it.Tq;
      const int tok_per_tile = kRows / group;
      const int tt0 = it.t0 + tile * tok_per_tile;       // first query token of the tile
      const int t = tt0 + r / group;                     // query token in the chunk
      const bool row_ok = t < Tq;
      // the row's output: out row, and the partition (-1: one partition,
      // direct; a shared prefix's partitions are always partials)
      const size_t orow = (size_t)(it.q0 + t) * num_q_heads + it.kvh * group + r % group;
      const int opart = it.n_parts == 1 && it.causal ? -1 : it.part;
      // last key this row may see
      const int lim = it.causal ? L - Tq + (row_ok ? t : 0) : L - 1;
      float m = -INFINITY, l = 0.f;                      // reference maximum (log2 units)
      // keys every row of the tile may see: up to the first row's causal limit
      const int key_all = it.causal ? min(key_end, L - Tq + tt0 + 1) : key_end;
      // Validity of the table entries of the step at key kb0 (a bit per cache
      // block), loaded one step ahead so the table reads never wait in the loop.
      auto bad_blocks = [&](int kb0) {
        const int32_t* bt_row = block_tables + (size_t)seq * bt_stride;
        int mask = 0;
#pragma unroll
        for (int b = 0; b < kStepBlocks; ++b) {
          const int lb = kb0 / 16 + b;
          if (lb * 16 < key_end) {
            const int p = __ldg(bt_row + lb);
            if (p < 0 || p >= num_blocks) mask |= 1 << b;
          }
        }
        return mask;
      };
      int bad_next = key_begin < key_end ? bad_blocks(key_begin) : 0;
      // one step per 128 keys; g counts steps over all items
      for (int kb = key_begin; kb < key_end; kb += kKeys, ++g) {
        const int st = g % kStages;
        const int bad_mask = bad_next;
        if (kb + kKeys < key_end) bad_next = bad_blocks(kb + kKeys);
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[tile], (uint32_t)(g & 1)))) { failed = true; break; }
        tc::fence_after_sync();
        float s[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) {
          float v[32];
          tc::tmem_ld32(lane_addr + (uint32_t)(c * 32), v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = v[i];
        }
        tc::tmem_wait_ld();
        // Logits in log2 units are s * scale_log2. Steps wholly inside the
        // tile's causal horizon need no mask (scale folded into the exp's FMA);
        // otherwise scale first and give masked keys -inf.
        const bool need_mask = kb + kKeys > key_all || bad_mask != 0;
        float mx, cc;
        if (need_mask) {
          mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < kKeys; ++i) {
            const int kp = kb + i;
            const bool ok = kp < key_end && kp <= lim && !((bad_mask >> (i >> 4)) & 1);
            s[i] = ok ? s[i] * scale_log2 : -INFINITY;
            mx = fmaxf(mx, s[i]);
          }
          cc = 1.f;
        } else {
          // the largest logit is the largest raw score (the smallest, for a
          // negative scale); four independent chains of three-input max
          static_assert(kKeys % 8 == 4 || kKeys % 8 == 0, "reduction layout");
          float e0 = s[0], e1 = s[1], e2 = s[2], e3 = s[3];
          if (scale_log2 >= 0.f) {
#pragma unroll
            for (int i = 4; i + 8 <= kKeys; i += 8) {
              e0 = max3(e0, s[i], s[i + 1]);
              e1 = max3(e1, s[i + 2], s[i + 3]);
              e2 = max3(e2, s[i + 4], s[i + 5]);
              e3 = max3(e3, s[i + 6], s[i + 7]);
            }
            e0 = max3(e0, s[kKeys - 4], s[kKeys - 3]);
            e1 = max3(e1, s[kKeys - 2], s[kKeys - 1]);
            mx = max3(e0, e1, fmaxf(e2, e3)) * scale_log2;
          } else {
#pragma unroll
            for (int i = 4; i + 8 <= kKeys; i += 8) {
              e0 = min3(e0, s[i], s[i + 1]);
              e1 = min3(e1, s[i + 2], s[i + 3]);
              e2 = min3(e2, s[i + 4], s[i + 5]);
              e3 = min3(e3, s[i + 6], s[i + 7]);
            }
            e0 = min3(e0, s[kKeys - 4], s[kKeys - 3]);
            e1 = min3(e1, s[kKeys - 2], s[kKeys - 1]);
            mx = min3(e0, e1, fminf(e2, e3)) * scale_log2;
          }
          cc = scale_log2;
        }
        float alpha = 1.f;
        if (mx > m + kRescaleLog2 || m == -INFINITY) {
          const float m_new = fmaxf(m, mx);
          alpha = m == -INFINITY ? 0.f : fast_exp2(m - m_new);
          m = m_new;
        }
        const float m_use = m == -INFINITY ? 0.f : m;
        // P_j row r: 128 bf16 = 64 columns over the S columns already read
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;  // four chains of row-sum adds
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(s[32 * c + 2 * i], cc, -m_use));
            const float p1 = fast_exp2(fmaf(s[32 * c + 2 * i + 1], cc, -m_use));
            if (i & 1) {
              sa1 += p0;
              sb1 += p1;
            } else {
              sa0 += p0;
              sb0 += p1;
            }
            pk[i] = E::pack(p0, p1);
          }
          tc::tmem_st16u(lane_addr + (uint32_t)(c * 16), pk);
        }
        l = l * alpha + ((sa0 + sa1) + (sb0 + sb1));
        // rescale O when a row's reference maximum moved (warp-uniform
        // decision; not at an item's first step, where P.V starts O afresh);
        // the previous step's P.V of this tile has completed (covered by
        // s_full's commit), this step's waits for this warp's p_ready arrival
        if (kb > key_begin && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
            float o[32];
            tc::tmem_ld32(lane_addr + kOCol + c * 32, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::tmem_st32(lane_addr + kOCol + c * 32, o);
          }
        }
        tc::tmem_wait_st();
        // V rows of keys past the context or of bad blocks become zero (once V
        // landed); tile 0 does it, before its p_ready, which the MMA warp awaits
        // before either tile's P.V of the step.
        if (tile == 0 && (kb + kKeys > key_end || bad_mask)) {
          if (!__all_sync(0xffffffffu, mbar_wait(&v_full[st], (uint32_t)((g / kStages) & 1)))) { failed = true; break; }
          uint8_t* v = stage_v(st);
          for (int i = r; i < kKeys * kChunks * 8; i += kRows) {
            const int c = i / (kKeys * 8), rem = i % (kKeys * 8);
            const int key = rem / 8;
            if (kb + key >= key_end || ((bad_mask >> (key >> 4)) & 1))
              *reinterpret_cast<uint4*>(v + c * (kKeys * 128) + key * 128 + (rem % 8) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();  // zeroed V rows -> visible to the tensor core
        }
        tc::fence_before_sync();
        mbar_arrive(&p_ready[tile]);
      }
      if (failed) break;
      // ---- the item's epilogue: O / l  ->  out (one partition) or fp32 partials
      const bool any = key_end > key_begin;  // the item had steps (and MMAs)
      if (any) {
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (uint32_t)(no & 1)))) { failed = true; break; }
        ++no;
        tc::fence_after_sync();
      }
      const bool direct = opart < 0;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        float o[32];
        if (any) {
          tc::tmem_ld32(lane_addr + kOCol + c * 32, o);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (row_ok) {
          if (direct) {
            uint4* dst = reinterpret_cast<uint4*>(out + orow * kD + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(E::pack(o[8 * v] * inv, o[8 * v + 1] * inv),
                                  E::pack(o[8 * v + 2] * inv, o[8 * v + 3] * inv),
                                  E::pack(o[8 * v + 4] * inv, o[8 * v + 5] * inv),
                                  E::pack(o[8 * v + 6] * inv, o[8 * v + 7] * inv));
          } else {
            float4* dst = reinterpret_cast<float4*>(part_o + (orow * max_parts + opart) * kD + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(o[4 * v] * inv, o[4 * v + 1] * inv, o[4 * v + 2] * inv,
                                   o[4 * v + 3] * inv);
          }
        }
      }
      if (row_ok && !direct)
        part_lse[orow * max_parts + opart] = l > 0.f ? m + log2f(l) : -INFINITY;
    }
    if (failed && lane == 0 && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
  }

  // ---- teardown: every thread done with TMEM, then warp 0 frees it
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  // A shared prefix's partitions run as a programmatic dependent of the
  // decode kernel that covers the other partitions, overlapping its end (the
  // two write disjoint partials; the inputs were complete before that kernel
  // started). This grid ends only after that one, so the reduce launched
  // after this grid, which waits for it, sees both.
  if (shared_L >= 0) griddep_wait();
}

// Longest-first order of the chunk kernel's work: the CTAs of a grid start in
// index order, so listing the (sequence, tile pair, partition) items by
// descending key steps makes the launch a longest-processing-time-first
// schedule, and the last wave ends with short items. One CTA: a histogram of
// the items' step counts (one bucket per thread), a descending scan, a
// scatter. An item is listed exactly when the kernel would do work (or count
// an error) for it; its step count is the kernel's n_steps.
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
    chunk_plan_kernel(const int32_t* __restrict__ context_lens,
                      const int32_t* __restrict__ q_start, int num_seqs, int num_q_tokens,
                      int max_query_len, int max_context_len, int group, int part_blocks,
                      int max_parts, uint2* __restrict__ items, int32_t* __restrict__ plan) {
  __shared__ int hist[kPlanThreads];
  __shared__ int cursor[kPlanThreads];
  __shared__ int warp_sum[kPlanThreads / 32];
  griddep_launch_dependents();  // the chunk kernel's CTAs may become resident now
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tok_per_tile = kRows / group;
  // visit(s, f): f(local item index, steps) for every item of sequence s
  auto visit = [&](int s, auto&& f) {
    int L = context_lens[s];
    L = L < 0 ? 0 : (L > max_context_len ? max_context_len : L);
    const int q0 = q_start[s];
    int Tq = q_start[s + 1] - q0;
    const bool bad_q = q0 < 0 || Tq < 0 || q0 + Tq > num_q_tokens;
    if (!bad_q) Tq = min(Tq, min(L, max_query_len));
    const int nblk = (L + 15) / 16;
    const int n_parts = nblk > 0 ? (nblk + part_blocks - 1) / part_blocks : 1;
    bool listed00 = false;
    if (!bad_q) {
      for (int t0 = 0, pair = 0; t0 < Tq; t0 += kTiles * tok_per_tile, ++pair) {
        const int t_last = min(t0 + kTiles * tok_per_tile, Tq) - 1;
        for (int p = 0; p < n_parts; ++p) {
          const int kb = p * part_blocks * 16;
          const int ke = min(min((p + 1) * part_blocks * 16, L), L - Tq + t_last + 1);
          const int steps = ke > kb ? (ke - kb + kKeys - 1) / kKeys : 0;
          f(pair * max_parts + p, steps);
          listed00 |= pair == 0 && p == 0;
        }
      }
    }
    // The kernel counts a sequence's argument errors in its first item: keep
    // that item even when it has no rows.
    if (!listed00) f(0, 0);
  };
  hist[tid] = 0;
  __syncthreads();
  for (int s = tid; s < num_seqs; s += kPlanThreads)
    visit(s, [&](int, int steps) { atomicAdd(&hist[min(steps, kPlanThreads - 1)], 1); });
  __syncthreads();
  // cursor[b] = items in buckets above b (more steps first)
  const int b = kPlanThreads - 1 - tid;
  const int v = hist[b];
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sum[lane] = w;
  }
  __syncthreads();
  const int incl = x + (warp > 0 ? warp_sum[warp - 1] : 0);
  cursor[b] = incl - v;
  if (tid == kPlanThreads - 1) {
    plan[0] = incl;  // items listed
    plan[1] = 0;     // work counter of the persistent chunk kernel
  }
  __syncthreads();
  for (int s = tid; s < num_seqs; s += kPlanThreads)
    visit(s, [&](int local, int steps) {
      items[atomicAdd(&cursor[min(steps, kPlanThreads - 1)], 1)] =
          make_uint2((unsigned)s, (unsigned)local);
    });
}

}  // namespace

bool prefill_tc_eligible(int32_t head_dim, int32_t group, int32_t max_query_len, int64_t parts,
                         int32_t partition_tokens) {
  const bool pow2 = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
  return head_dim == kD && pow2 && (int64_t)max_query_len * group >= 64 &&
         (parts <= 1 || partition_tokens % kKeys == 0);
}

int64_t prefill_tc_max_items(int32_t num_seqs, int32_t max_query_len, int32_t group,
                             int64_t parts) {
  const int64_t tiles = ((int64_t)max_query_len * group + kRows - 1) / kRows;
  const int64_t pairs = (tiles + kTiles - 1) / kTiles;
  return (int64_t)num_seqs * (pairs > 0 ? pairs : 1) * (parts > 0 ? parts : 1);
}

bool prefill_tc_supported(const DecodeLaunch& a) {
  const int g = a.group;
  return a.q_start && a.head_dim == kD && (g == 1 || g == 2 || g == 4 || g == 8 || g == 16) &&
         (a.max_parts == 1 || (a.part_tokens % kKeys) == 0);
}

cudaError_t launch_prefill_tc(const DecodeLaunch& a, const CUtensorMap& tm_q,
                              cudaStream_t stream) {
  auto run = [&](auto* tag) -> cudaError_t {
    using T = std::remove_pointer_t<decltype(tag)>;
    auto kern = prefill_tc_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemAlloc);
    if (e != cudaSuccess) return e;
    const int qtiles = (a.max_query_len * a.group + kRows - 1) / kRows;
    const int pairs = (qtiles + kTiles - 1) / kTiles;
    if (!a.chunk_plan) {
      dim3 grid((unsigned)((int64_t)a.max_parts * pairs), a.num_kv_heads, a.num_seqs);
      kern<<<grid, kThreadsTc, kSmemAlloc, stream>>>(
          tm_q, a.tm_k, a.tm_v, static_cast<T*>(a.out), a.part_o, a.part_lse, a.q_start,
          a.num_q_tokens, a.max_query_len, a.block_tables, a.bt_stride, a.context_lens,
          a.num_q_heads, a.group, a.num_blocks, a.max_context_len, a.scale_log2, a.part_blocks,
          a.max_parts, a.dev_error, nullptr, nullptr, a.num_kv_heads, -1);
      return cudaGetLastError();
    }
    // Longest first: the plan kernel lists the items and zeroes the work
    // counter; the chunk kernel (a programmatic dependent: resident while the
    // plan runs, reading nothing before griddepcontrol.wait) runs one CTA per
    // SM, each taking the next item of the list from the counter when it is
    // ready for one.
    const int64_t n_max = prefill_tc_max_items(a.num_seqs, a.max_query_len, a.group,
                                               a.max_parts) * a.num_kv_heads;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t ctas = n_max < (int64_t)sms ? n_max : (int64_t)sms;  // one CTA per SM fits
    chunk_plan_kernel<<<1, kPlanThreads, 0, stream>>>(
        a.context_lens, a.q_start, a.num_seqs, a.num_q_tokens, a.max_query_len,
        a.max_context_len, a.group, a.part_blocks, a.max_parts, a.chunk_items, a.chunk_plan);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ctas > 0 ? ctas : 1));
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tm_q, a.tm_k, a.tm_v, static_cast<T*>(a.out), a.part_o,
                              a.part_lse, a.q_start, a.num_q_tokens, a.max_query_len,
                              a.block_tables, a.bt_stride, a.context_lens, a.num_q_heads,
                              a.group, a.num_blocks, a.max_context_len, a.scale_log2,
                              a.part_blocks, a.max_parts, a.dev_error,
                              static_cast<const uint2*>(a.chunk_items),
                              a.chunk_plan, a.num_kv_heads, -1);
  };
  return a.bf16 ? run((__nv_bfloat16*)nullptr) : run((__half*)nullptr);
}

bool prefill_tc_shared_supported(const DecodeLaunch& a) {
  const int g = a.group;
  return !a.q_start && a.head_dim == kD && (g == 1 || g == 2 || g == 4 || g == 8 || g == 16) &&
         (int64_t)a.num_q_tokens * g >= 64 && a.part_tokens % kKeys == 0 && a.first_part >= 1 &&
         a.first_part < a.max_parts && a.part_o && a.part_lse;
}

cudaError_t launch_prefill_tc_shared(const DecodeLaunch& a, const CUtensorMap& tm_q,
                                     cudaStream_t stream) {
  auto run = [&](auto* tag) -> cudaError_t {
    using T = std::remove_pointer_t<decltype(tag)>;
    auto kern = prefill_tc_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemAlloc);
    if (e != cudaSuccess) return e;
    // one virtual sequence: all rows of q as its query tokens; its items are
    // (tile pair, partition < first_part, KV head), grid order
    const int64_t qtiles = ((int64_t)a.num_q_tokens * a.group + kRows - 1) / kRows;
    const int64_t pairs = (qtiles + kTiles - 1) / kTiles;
    const int shared_L = a.first_part * a.part_tokens;
    // a programmatic dependent of the decode kernel launched before it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.max_parts * pairs), a.num_kv_heads, 1);
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tm_q, a.tm_k, a.tm_v, static_cast<T*>(a.out),
                              a.part_o, a.part_lse, static_cast<const int32_t*>(nullptr),
                              a.num_q_tokens, a.num_q_tokens, a.block_tables, a.bt_stride,
                              static_cast<const int32_t*>(nullptr), a.num_q_heads, a.group,
                              a.num_blocks, a.max_context_len, a.scale_log2, a.part_blocks,
                              a.max_parts, a.dev_error, static_cast<const uint2*>(nullptr),
                              static_cast<int32_t*>(nullptr), a.num_kv_heads, shared_L);
  };
  return a.bf16 ? run((__nv_bfloat16*)nullptr) : run((__half*)nullptr);
}

}  // namespace pa
