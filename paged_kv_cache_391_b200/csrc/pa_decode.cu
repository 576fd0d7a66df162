// pa_decode.cu -- paged single-token decode attention for sm_100a.
//
// What it computes ("Optimizing LLM Inference: From PagedAttention to AI
// Infra", "PagedAttention: Decoupling Logical Context from Contiguous GPU
// Memory", Figure 2; "The Memory Wall ...", "How it Works Under the Hood" and
// "Show Me The Code"): for every sequence s and query head h,
//     out[s][h] = sum_t softmax_t(scale * <q[s][h], K_t>) V_t
// over the context's tokens, found by walking the block table in logical
// order. Long contexts are split into fixed token partitions ("PagedAttention
// in Action ...", "New Developments in 2026": sequence splits as a unit of
// decode scheduling) whose results a log-sum-exp reduce combines.
//
// Design (B200):
//  * One CTA per (partition, KV head, sequence); its four warps take the
//    partition's 16-token blocks round-robin, each with a private 2-stage ring
//    of shared-memory tiles (three CTAs per SM keep ~24 tiles in flight). A tile (one block, one KV head: 16 x D values,
//    contiguous in HBM) arrives by TMA as 64-column boxes with a 128-byte
//    swizzle, so the ldmatrix reads below are bank-conflict free. Completion
//    is tracked by one mbarrier per stage; every wait is bounded.
//  * All query heads of a KV head share each K/V load (GQA). q.K^T and P.V
//    run on the tensor cores as m16n8k16 tiles with the query heads as the M
//    dimension (up to 16), tokens and head-dim columns as N and K; the P tile
//    is taken straight from the q.K^T accumulators without a shuffle.
//  * Softmax is online, per warp, in fp32 and base 2 (scale * log2 e folded
//    into one multiply); the four warps and then the partitions are merged by
//    log-sum-exp. Tokens past the context are masked to -inf and their V rows
//    zeroed in shared memory, so stale cache contents never reach the output.
//  * The arithmetic follows logical token order only, so the output does not
//    depend on which physical blocks hold the context, bit for bit.
#include <math.h>

#include <utility>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// CTA shape: warps per CTA and shared-memory stages per warp (compile-time).
// 4 warps x 2 stages = 64 KiB of tiles per CTA, three CTAs per SM: measured on
// B200 to beat deeper rings with fewer resident CTAs (2 or 1 per SM), because
// the CTAs' start-up and merge phases then overlap other CTAs' streaming.
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif

constexpr int kBlockTokens = 16;
constexpr int kWarps = PA_DECODE_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct DecodeSmem {
  static constexpr int kStages = PA_DECODE_STAGES;
  static constexpr int kSubTiles = D / 64;                 // 128-byte TMA boxes per tile
  static constexpr int kTileBytes = kBlockTokens * D * 2;  // K (or V) of one block, one KV head
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kTileRegion = kWarps * kWarpBytes;
  static constexpr int kBarOffset = kTileRegion;
  static constexpr int kBytes = kTileRegion + kWarps * kStages * 8;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static constexpr int kMergeStride = D + 8;    // floats per (warp, head) row of the merge
  static_assert(kWarps * 16 * kMergeStride * 4 + 2 * kWarps * 16 * 4 <= kTileRegion,
                "merge scratch must fit in the tile region");
};

// Byte offset of element (token t, column d) inside one swizzled tile: the
// tile is D/64 boxes of 16 rows x 128 bytes, and the 16-byte chunk index
// within a row is XORed with (row % 8), as TMA's 128-byte swizzle lays it out.
__device__ __forceinline__ uint32_t tile_off(int t, int d) {
  return (uint32_t)((d >> 6) * 2048 + t * 128 + ((((d & 63) >> 3) ^ (t & 7)) << 4) + (d & 7) * 2);
}

// The arguments every work item shares.
template <typename T>
struct ItemArgs {
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
  T* out;
  float* part_o;
  float* part_lse;
  const T* q;
  const int32_t* q_start;
  int num_q_tokens, max_query_len;
  const int32_t* block_tables;
  int bt_stride;
  const int32_t* context_lens;
  int num_q_heads, group;
  int64_t num_blocks;
  int max_context_len;
  float scale_log2;
  int part_blocks, max_parts;
  int32_t* dev_error;
};

// One work item: (partition, KV head, sequence, query tile), by the whole CTA.
// kMulti = false: one query token per sequence (decode); the tile's rows are
// the query heads of one KV head. kMulti = true: each sequence's last Tq
// context tokens are queries (a prompt chunk, or speculative draft tokens);
// the tile's rows are (query token, head) pairs, 16 per tile, and query token
// t sees the context up to its own position L - Tq + t (causal in the chunk).
// `ring` counts the tiles this warp has consumed from its ring before the
// item (stage and mbarrier parity continue from it across items); with
// init_bars the warp first initialises its ring's barriers. Returns true if a
// tile wait ran out of time (the error is counted in dev_error).
template <typename T, int D, bool kTwoRows, bool kMulti>
__device__ __forceinline__ bool attend_item(const ItemArgs<T>& A, uint8_t* smem, uint64_t* bars,
                                            int part, int kvh, int seq, int qtile,
                                            bool init_bars, uint32_t& ring) {
  using SM = DecodeSmem<D>;
  using E = Elem<T>;
  const CUtensorMap* tm_k = A.tm_k;
  const CUtensorMap* tm_v = A.tm_v;
  T* __restrict__ out = A.out;
  float* __restrict__ part_o = A.part_o;
  float* __restrict__ part_lse = A.part_lse;
  const T* __restrict__ q = A.q;
  const int32_t* __restrict__ q_start = A.q_start;
  const int num_q_tokens = A.num_q_tokens, max_query_len = A.max_query_len;
  const int32_t* __restrict__ block_tables = A.block_tables;
  const int bt_stride = A.bt_stride;
  const int32_t* __restrict__ context_lens = A.context_lens;
  const int num_q_heads = A.num_q_heads, group = A.group;
  const int64_t num_blocks = A.num_blocks;
  const int max_context_len = A.max_context_len;
  const float scale_log2 = A.scale_log2;
  const int part_blocks = A.part_blocks, max_parts = A.max_parts;
  int32_t* __restrict__ dev_error = A.dev_error;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const bool counter = part == 0 && kvh == 0 && qtile == 0 && tid == 0 && dev_error;

  int L = context_lens[seq];
  if (L < 0 || L > max_context_len) {
    if (counter) atomicAdd(dev_error, 1);
    L = L < 0 ? 0 : max_context_len;
  }
  // Query rows of this sequence: q0 = first query token, Tq tokens.
  int q0 = seq, Tq = 1;
  if (kMulti) {
    q0 = q_start[seq];
    Tq = q_start[seq + 1] - q0;
    if (q0 < 0 || Tq < 0 || q0 + Tq > num_q_tokens) {
      if (counter) atomicAdd(dev_error, 1);  // query range outside the q buffer: skip
      return false;
    }
    const int cap = min(L, max_query_len);
    if (Tq > cap) {
      if (counter) atomicAdd(dev_error, 1);
      Tq = cap;
    }
  }
  const int rows_total = Tq * group;
  const int row0 = qtile * 16;
  if (row0 >= rows_total) return false;
  const int nrows = min(16, rows_total - row0);  // rows of this tile (decode: = group)

  const int nblk_seq = (L + kBlockTokens - 1) / kBlockTokens;
  const int n_parts = nblk_seq > 0 ? (nblk_seq + part_blocks - 1) / part_blocks : 1;
  if (part >= n_parts) return false;
  const int blk_begin = part * part_blocks;
  const int nblk = min(nblk_seq - blk_begin, part_blocks);  // 0 only for an empty context
  const int q_head0 = kvh * group;
  // This lane's two tile rows (a = gid, b = gid + 8): query token and head.
  const int ta = (row0 + gid) / group, ha = (row0 + gid) - ta * group;
  const int tb = (row0 + gid + 8) / group, hb = (row0 + gid + 8) - tb * group;
  const int lim_a = L - Tq + ta;  // last key position row a may attend to
  const int lim_b = L - Tq + tb;

  // ---- this warp's share: blocks blk_begin + warp + kWarps * it
  const int n_mine = nblk > warp ? (nblk - warp + kWarps - 1) / kWarps : 0;
  uint8_t* wtiles = smem + warp * SM::kWarpBytes;
  uint64_t* wbars = bars + warp * SM::kStages;
  if (init_bars) {
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < SM::kStages; ++s) mbar_init(&wbars[s], 1);
      fence_barrier_init();
      if (warp == 0) {
        tma_prefetch_desc(tm_k);
        tma_prefetch_desc(tm_v);
      }
    }
    __syncwarp();
  }

  // Physical block ids, 32 iterations per register window; ids outside the
  // pool are skipped and counted once (by the KV-head-0 CTA of the first
  // query tile: every query tile's CTA reads the partition's whole table).
  const int32_t* bt_mine = block_tables + (size_t)seq * bt_stride + blk_begin + warp;
  auto load_pid = [&](int it) -> int {
    int p = -1;
    if (it < n_mine) {
      p = __ldg(bt_mine + kWarps * it);
      if (p < 0 || p >= num_blocks) {
        if (kvh == 0 && qtile == 0 && dev_error) atomicAdd(dev_error, 1);
        p = -1;
      }
    }
    return p;
  };
  int win = 0;
  int pid_cur = load_pid(lane);
  int pid_nxt = load_pid(32 + lane);
  auto pid_of = [&](int it) -> int {
    const int v = ((it >> 5) == win) ? pid_cur : pid_nxt;
    return __shfl_sync(kFull, v, it & 31);
  };
  auto issue = [&](int it, int p) {  // lane 0 only
    const int st = (ring + it) % SM::kStages;
    uint8_t* kt = wtiles + st * SM::kStageBytes;
    uint8_t* vt = kt + SM::kTileBytes;
    if (p >= 0) {
      mbar_arrive_expect_tx(&wbars[st], 2 * SM::kTileBytes);
#pragma unroll
      for (int c = 0; c < SM::kSubTiles; ++c) {
        tma_load_4d(kt + c * 2048, tm_k, &wbars[st], c * 64, 0, kvh, p);
        tma_load_4d(vt + c * 2048, tm_v, &wbars[st], c * 64, 0, kvh, p);
      }
    } else {
      mbar_arrive(&wbars[st]);  // nothing to load: complete the phase empty
    }
  };
  {
    const int n_pro = min(n_mine, SM::kStages);
    for (int it = 0; it < n_pro; ++it) {
      const int p = pid_of(it);
      if (lane == 0) issue(it, p);
    }
  }

  // ---- query fragments (A operand of q.K^T): rows = heads of this group
  uint32_t qa[D / 16][4];
  {
    const uint32_t* qa_row =
        gid < nrows ? reinterpret_cast<const uint32_t*>(
                          q + ((size_t)(q0 + ta) * num_q_heads + q_head0 + ha) * D)
                    : nullptr;
    const uint32_t* qb_row =
        (kTwoRows && gid + 8 < nrows)
            ? reinterpret_cast<const uint32_t*>(q + ((size_t)(q0 + tb) * num_q_heads + q_head0 + hb) * D)
            : nullptr;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qa[kk][0] = qa_row ? __ldg(qa_row + kk * 8 + tig) : 0u;
      qa[kk][1] = qb_row ? __ldg(qb_row + kk * 8 + tig) : 0u;
      qa[kk][2] = qa_row ? __ldg(qa_row + kk * 8 + 4 + tig) : 0u;
      qa[kk][3] = qb_row ? __ldg(qb_row + kk * 8 + 4 + tig) : 0u;
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  const int mi = lane >> 3, r8 = lane & 7;
  int it = 0;
  bool timed_out = false;
  for (; it < n_mine; ++it) {
    if (it > 0 && (it & 31) == 0) {
      ++win;
      pid_cur = pid_nxt;
      pid_nxt = load_pid((win + 1) * 32 + lane);
    }
    const int st = (ring + it) % SM::kStages;
    const uint32_t parity = (uint32_t)(((ring + it) / SM::kStages) & 1);
    const int p = pid_of(it);
    if (!__all_sync(kFull, mbar_wait_tile(&wbars[st], parity))) {
      timed_out = true;
      break;
    }
    if (p >= 0) {
      uint8_t* kt = wtiles + st * SM::kStageBytes;
      uint8_t* vt = kt + SM::kTileBytes;
      const int j = blk_begin + warp + kWarps * it;
      const int valid = min(kBlockTokens, L - j * kBlockTokens);
      if (valid < kBlockTokens) {
        // Zero the V rows past the context: P is 0 there, and 0 * NaN would not be.
        const int nrow = kBlockTokens - valid;
        for (int i = lane; i < nrow * SM::kSubTiles * 8; i += 32) {
          const int c = i / (nrow * 8), rem = i % (nrow * 8);
          *reinterpret_cast<uint4*>(vt + c * 2048 + (valid + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }

      // S = Q K^T for the 16 tokens: two n-tiles of 8 tokens, K over D; the
      // even and odd K steps accumulate separately (two dependency chains of
      // D/32 tensor-core ops instead of one of D/16), then add.
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
      float u0[4] = {0.f, 0.f, 0.f, 0.f}, u1[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kbase = smem_addr(kt);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + tile_off((mi >> 1) * 8 + r8, kk * 16 + (mi & 1) * 8), b0, b1, b2, b3);
        if (kk & 1) {
          E::mma(u0, qa[kk], b0, b1);
          E::mma(u1, qa[kk], b2, b3);
        } else {
          E::mma(s0, qa[kk], b0, b1);
          E::mma(s1, qa[kk], b2, b3);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s0[i] += u0[i];
        s1[i] += u1[i];
      }

      // Online softmax (base 2). Lane holds, for head row a = gid (and
      // b = gid + 8), tokens 2tig, 2tig+1 (s0) and 8+2tig, 9+2tig (s1).
      // Keys of this block row a (b) may see: the context, and in a chunk
      // only up to the row's own position.
      const int t0 = 2 * tig;
      const int na = kMulti ? min(valid, lim_a - j * kBlockTokens + 1) : valid;
      const int nb = kMulti ? min(valid, lim_b - j * kBlockTokens + 1) : valid;
      bool v0 = t0 < na, v1 = t0 + 1 < na, v2 = t0 + 8 < na, v3 = t0 + 9 < na;
      uint32_t pa[4];
      {
        const float x0 = v0 ? s0[0] * scale_log2 : -INFINITY;
        const float x1 = v1 ? s0[1] * scale_log2 : -INFINITY;
        const float x2 = v2 ? s1[0] * scale_log2 : -INFINITY;
        const float x3 = v3 ? s1[1] * scale_log2 : -INFINITY;
        float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m_a, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = exp2f(m_a - m_use);
        pa[0] = E::pack(exp2f(x0 - m_use), exp2f(x1 - m_use));
        pa[2] = E::pack(exp2f(x2 - m_use), exp2f(x3 - m_use));
        const float2 u0 = E::unpack(pa[0]), u2 = E::unpack(pa[2]);
        l_a = l_a * alpha + ((u0.x + u0.y) + (u2.x + u2.y));
        m_a = m_new;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= alpha;
          o[n][1] *= alpha;
        }
      }
      if (kTwoRows) {
        v0 = t0 < nb, v1 = t0 + 1 < nb, v2 = t0 + 8 < nb, v3 = t0 + 9 < nb;
        const float x0 = v0 ? s0[2] * scale_log2 : -INFINITY;
        const float x1 = v1 ? s0[3] * scale_log2 : -INFINITY;
        const float x2 = v2 ? s1[2] * scale_log2 : -INFINITY;
        const float x3 = v3 ? s1[3] * scale_log2 : -INFINITY;
        float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m_b, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = exp2f(m_b - m_use);
        pa[1] = E::pack(exp2f(x0 - m_use), exp2f(x1 - m_use));
        pa[3] = E::pack(exp2f(x2 - m_use), exp2f(x3 - m_use));
        const float2 u1 = E::unpack(pa[1]), u3 = E::unpack(pa[3]);
        l_b = l_b * alpha + ((u1.x + u1.y) + (u3.x + u3.y));
        m_b = m_new;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][2] *= alpha;
          o[n][3] *= alpha;
        }
      } else {
        pa[1] = 0u;
        pa[3] = 0u;
      }

      // O += P V: N = head-dim columns (pairs of 8-column n-tiles), K = 16 tokens.
      const uint32_t vbase = smem_addr(vt);
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vbase + tile_off((mi & 1) * 8 + r8, n2 * 16 + (mi >> 1) * 8), b0, b1, b2,
                      b3);
        E::mma(o[2 * n2], pa, b0, b1);
        E::mma(o[2 * n2 + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (it + SM::kStages < n_mine) {
      const int pn = pid_of(it + SM::kStages);
      if (lane == 0) issue(it + SM::kStages, pn);
    }
  }
  if (timed_out) {
    // Let the copies already in flight (tiles it .. it + kStages - 1) land,
    // each wait bounded, before the shared memory is reused or the CTA exits,
    // then report. The ring advances by the phases that completed.
    const int last = min(n_mine, it + SM::kStages);
    for (int k = it; k < last; ++k)
      (void)mbar_wait(&wbars[(ring + k) % SM::kStages], ((ring + k) / SM::kStages) & 1);
    if (lane == 0 && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
    ring += (uint32_t)last;
  } else {
    ring += (uint32_t)n_mine;
  }

  // ---- merge the four warps (log-sum-exp), then write out or the partials
  l_a += __shfl_xor_sync(kFull, l_a, 1);
  l_a += __shfl_xor_sync(kFull, l_a, 2);
  if (kTwoRows) {
    l_b += __shfl_xor_sync(kFull, l_b, 1);
    l_b += __shfl_xor_sync(kFull, l_b, 2);
  }
  __syncthreads();  // every warp is done with its tiles
  float* mo = reinterpret_cast<float*>(smem);
  float* mm = mo + kWarps * 16 * SM::kMergeStride;
  float* ml = mm + kWarps * 16;
  if (gid < nrows) {
    float* row = mo + (warp * 16 + gid) * SM::kMergeStride;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<float2*>(row + n * 8 + 2 * tig) = make_float2(o[n][0], o[n][1]);
    if (tig == 0) {
      mm[warp * 16 + gid] = m_a;
      ml[warp * 16 + gid] = l_a;
    }
  }
  if (kTwoRows && gid + 8 < nrows) {
    float* row = mo + (warp * 16 + gid + 8) * SM::kMergeStride;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<float2*>(row + n * 8 + 2 * tig) = make_float2(o[n][2], o[n][3]);
    if (tig == 0) {
      mm[warp * 16 + gid + 8] = m_b;
      ml[warp * 16 + gid + 8] = l_b;
    }
  }
  __syncthreads();

  const bool direct = n_parts == 1;
  for (int idx = tid; idx < nrows * (D / 4); idx += kThreads) {
    const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;  // h: tile row
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * 16 + h]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float sc = exp2f(mm[w * 16 + h] - M);
        lsum += ml[w * 16 + h] * sc;
        const float4 v = *reinterpret_cast<const float4*>(mo + (w * 16 + h) * SM::kMergeStride + d);
        acc.x += sc * v.x;
        acc.y += sc * v.y;
        acc.z += sc * v.z;
        acc.w += sc * v.w;
      }
    }
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lsum > 0.f) {
      res.x = acc.x / lsum;
      res.y = acc.y / lsum;
      res.z = acc.z / lsum;
      res.w = acc.w / lsum;
    }
    const int t = (row0 + h) / group;
    const size_t orow = (size_t)(q0 + t) * num_q_heads + q_head0 + (row0 + h - t * group);
    if (direct) {
      uint2 pk;
      pk.x = E::pack(res.x, res.y);
      pk.y = E::pack(res.z, res.w);
      *reinterpret_cast<uint2*>(out + orow * D + d) = pk;
    } else {
      *reinterpret_cast<float4*>(part_o + (orow * max_parts + part) * D + d) = res;
      if (d == 0) part_lse[orow * max_parts + part] = lsum > 0.f ? M + log2f(lsum) : -INFINITY;
    }
  }
  return timed_out;
}

// One CTA per work item: grid (max_parts * query tiles, KV heads, sequences).
template <typename T, int D, bool kTwoRows, bool kMulti>
__global__ void __launch_bounds__(kThreads)
    decode_partition_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, T* __restrict__ out,
                            float* __restrict__ part_o, float* __restrict__ part_lse,
                            const T* __restrict__ q, const int32_t* __restrict__ q_start,
                            int num_q_tokens, int max_query_len,
                            const int32_t* __restrict__ block_tables, int bt_stride,
                            const int32_t* __restrict__ context_lens, int num_q_heads, int group,
                            int64_t num_blocks, int max_context_len, float scale_log2,
                            int part_blocks, int max_parts, int32_t* __restrict__ dev_error,
                            int first_part) {
  using SM = DecodeSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOffset);
  const ItemArgs<T> A{&tm_k,        &tm_v,     out,          part_o,        part_lse,
                      q,            q_start,   num_q_tokens, max_query_len, block_tables,
                      bt_stride,    context_lens, num_q_heads, group,       num_blocks,
                      max_context_len, scale_log2, part_blocks, max_parts,  dev_error};
  // first_part > 0 (decode only): the partitions below it, the shared
  // prefix's, were computed by another kernel.
  const int part = kMulti ? (int)(blockIdx.x % (unsigned)max_parts) : (int)blockIdx.x + first_part;
  const int qtile = kMulti ? (int)(blockIdx.x / (unsigned)max_parts) : 0;
  // Launched as a programmatic dependent: the CTA is resident when the
  // previous kernel ends, and waits for it before any read (empty
  // partitions then exit before setting up barriers).
  griddep_wait();
  if (!kMulti && first_part > 0 && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 32 &&
      dev_error) {
    // The prefix partitions assumed every sequence's table to start with
    // sequence 0's first first_part * part_blocks entries and its context to
    // cover them: a sequence for which that is false is counted (once; its
    // output is then not its attention).
    const int s = blockIdx.z, lane = threadIdx.x;
    const int pre = first_part * part_blocks;
    bool bad = false;
    if (lane == 0) {
      const int L = context_lens[s];
      bad = L < pre * 16 || L > max_context_len;
    }
    const int32_t* row = block_tables + (size_t)s * bt_stride;
    for (int i = lane; i < pre && s > 0; i += 32) bad |= row[i] != block_tables[i];
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicAdd(dev_error, 1);
  }
  // With a shared prefix the next kernel, the prefix's partitions, reads
  // nothing this one writes: it may start on the SMs this grid leaves free.
  if (!kMulti && first_part > 0) griddep_launch_dependents();
  uint32_t ring = 0;
  (void)attend_item<T, D, kTwoRows, kMulti>(A, smem, bars, part, blockIdx.y, blockIdx.z, qtile,
                                            true, ring);
}

// ---------------------------------------------------------------- work queue
// Page-aware decode scheduling ("New Developments in 2026", PersistentKV:
// pages, KV-head groups, sequence splits and work queues): a plan kernel
// lists the (sequence, partition) items, longest first, and a persistent grid
// of one wave of CTAs pulls (item, KV head) pairs from a global counter.
// Empty partitions of short sequences cost nothing, and the long items start
// first, so the last wave's tail is one short item.
//
// Plan layout (workspace): items[num_seqs * max_parts] = (seq << 16) | part,
// then plan[0] = number of items, plan[1] = the work counter (zeroed here).
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 1024;  // item length in blocks, clamped; one bucket per thread

__device__ __forceinline__ void plan_counts(const int32_t* context_lens, int s,
                                            int max_context_len, int part_blocks, int& n,
                                            int& tail_blocks) {
  int L = context_lens[s];
  L = L < 0 ? 0 : (L > max_context_len ? max_context_len : L);  // as attend_item clamps
  const int nblk = (L + kBlockTokens - 1) / kBlockTokens;
  n = nblk > 0 ? (nblk + part_blocks - 1) / part_blocks : 1;
  tail_blocks = nblk - (n - 1) * part_blocks;  // 0 for an empty context
}

__global__ void __launch_bounds__(kPlanThreads)
    decode_plan_kernel(const int32_t* __restrict__ context_lens, int num_seqs,
                       int max_context_len, int part_blocks, uint32_t* __restrict__ items,
                       int32_t* __restrict__ plan) {
  static_assert(kPlanThreads == kPlanBuckets, "one scan element per thread");
  __shared__ int hist[kPlanBuckets];
  __shared__ int cursor[kPlanBuckets];
  __shared__ int warp_sum[kPlanThreads / 32];
  griddep_launch_dependents();  // the decode grid may start its prologue now
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int full_bucket = min(part_blocks, kPlanBuckets - 1);
  hist[tid] = 0;
  __syncthreads();
  for (int s = tid; s < num_seqs; s += kPlanThreads) {
    int n, tail;
    plan_counts(context_lens, s, max_context_len, part_blocks, n, tail);
    if (n > 1) atomicAdd(&hist[full_bucket], n - 1);
    atomicAdd(&hist[min(tail, kPlanBuckets - 1)], 1);
  }
  __syncthreads();
  // cursor[b] = items in buckets above b (longer items first): an inclusive
  // scan over the reversed bucket order, minus the bucket's own count.
  const int b = kPlanBuckets - 1 - tid;
  const int v = hist[b];
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    warp_sum[lane] = w;
  }
  __syncthreads();
  const int incl = x + (warp > 0 ? warp_sum[warp - 1] : 0);
  cursor[b] = incl - v;
  if (tid == kPlanThreads - 1) {
    plan[0] = incl;  // all items
    plan[1] = 0;     // work counter
  }
  __syncthreads();
  for (int s = tid; s < num_seqs; s += kPlanThreads) {
    int n, tail;
    plan_counts(context_lens, s, max_context_len, part_blocks, n, tail);
    const uint32_t key = (uint32_t)s << 16;
    if (n > 1) {
      const int base = atomicAdd(&cursor[full_bucket], n - 1);
      for (int p = 0; p < n - 1; ++p) items[base + p] = key | (uint32_t)p;
    }
    items[atomicAdd(&cursor[min(tail, kPlanBuckets - 1)], 1)] = key | (uint32_t)(n - 1);
  }
}

// One wave of CTAs; each pulls work w -> (items[w / H_kv], KV head w % H_kv)
// until the plan's items run out. A CTA's first work is its own index; each
// later one comes from the counter, fetched one item ahead so the atomic's
// latency hides behind the current item.
template <typename T, int D, bool kTwoRows>
__global__ void __launch_bounds__(kThreads)
    decode_persistent_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, T* __restrict__ out,
                             float* __restrict__ part_o, float* __restrict__ part_lse,
                             const T* __restrict__ q, const int32_t* __restrict__ block_tables,
                             int bt_stride, const int32_t* __restrict__ context_lens,
                             int num_seqs, int num_q_heads, int group, int num_kv_heads,
                             int64_t num_blocks, int max_context_len, float scale_log2,
                             int part_blocks, int max_parts, const uint32_t* __restrict__ items,
                             int32_t* __restrict__ plan, int32_t* __restrict__ dev_error) {
  using SM = DecodeSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_next[2];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOffset);
  const ItemArgs<T> A{&tm_k,        &tm_v,     out,      part_o,        part_lse,
                      q,            nullptr,   num_seqs, 1,             block_tables,
                      bt_stride,    context_lens, num_q_heads, group,   num_blocks,
                      max_context_len, scale_log2, part_blocks, max_parts, dev_error};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < SM::kStages; ++s) mbar_init(&bars[warp * SM::kStages + s], 1);
    fence_barrier_init();
    if (warp == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
  }
  __syncwarp();
  griddep_wait();  // the plan is complete and visible from here on

  const int n_work = plan[0] * num_kv_heads;
  int32_t* counter = plan + 1;
  uint32_t ring = 0;
  int w = blockIdx.x;
  for (int k = 0; w < n_work; ++k) {
    int nxt = 0;
    if (threadIdx.x == 0) nxt = (int)gridDim.x + atomicAdd(counter, 1);
    const uint32_t it = items[w / num_kv_heads];
    const int seq = (int)(it >> 16), part = (int)(it & 0xffffu);
    bool timed_out = false;
    if (seq < num_seqs)
      timed_out = attend_item<T, D, kTwoRows, false>(A, smem, bars, part, w % num_kv_heads, seq,
                                                     0, false, ring);
    // The item's generic shared-memory accesses (merge scratch, zeroed V
    // rows) come before the next item's TMA writes to the same bytes.
    fence_proxy_async_smem();
    if (threadIdx.x == 0) s_next[k & 1] = nxt;
    if (__syncthreads_or(timed_out)) break;
    w = s_next[k & 1];
  }
}

// Combine the partitions of each (sequence, query head) row:
//   out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M),  M = max_p lse_p.
// Two phases, so the partial loads do not wait on each other: the weights
// first (max and sum in a fixed order), then independent weighted loads.
// Deterministic: the summation order depends only on the partition count.
constexpr int kReduceWarps = 8;

// Sequence of an output row: rows are (query token, head); with one token per
// sequence the token is the sequence, otherwise q_start (the first token of
// each sequence, num_seqs + 1 entries) is searched.
__device__ __forceinline__ int seq_of_row(int row, int num_q_heads, const int32_t* q_start,
                                          int num_seqs) {
  const int token = row / num_q_heads;
  if (!q_start) return token;
  int lo = 0, hi = num_seqs - 1;  // last seq with q_start[seq] <= token
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q_start[mid] <= token) lo = mid; else hi = mid - 1;
  }
  return lo;
}
constexpr int kWarpRowMaxParts = 16;  // up to this many, one warp (half-warp) per row

// Rows of up to kWarpRowMaxParts partitions: a warp (half-warp at D = 64)
// per row, kReduceWarps rows per CTA; `cta` is this CTA's index among them.
template <typename T, int D>
__device__ __forceinline__ void reduce_rows_warp(T* __restrict__ out,
                                                 const float* __restrict__ part_o,
                                                 const float* __restrict__ part_lse,
                                                 const int32_t* __restrict__ context_lens,
                                                 const int32_t* __restrict__ q_start,
                                                 int num_seqs, int num_rows, int num_q_heads,
                                                 int max_context_len, int part_tokens,
                                                 int max_parts, int cta) {
  constexpr int kLanes = D / 4;             // float4 columns of a row = lanes per row
  constexpr int kRowsPerWarp = 32 / kLanes;
  using E = Elem<T>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = (cta * kReduceWarps + warp) * kRowsPerWarp + lane / kLanes;
  const int c = lane % kLanes;
  const unsigned grp = kRowsPerWarp == 1 ? kFull : (0xffffu << (lane & ~(kLanes - 1)));
  int n = 0;
  if (row < num_rows) {
    int L = context_lens[seq_of_row(row, num_q_heads, q_start, num_seqs)];
    L = L < 0 ? 0 : (L > max_context_len ? max_context_len : L);
    n = (L + part_tokens - 1) / part_tokens;
  }
  // n is uniform within a row's lane group; rows with n <= 1 were written
  // directly, rows with more than kWarpRowMaxParts go to the split kernel
  if (n <= 1 || n > kWarpRowMaxParts) return;
  const float* lse = part_lse + (size_t)row * max_parts;
  const float4* po = reinterpret_cast<const float4*>(part_o + (size_t)row * max_parts * D);

  const float my_lse = c < n ? lse[c] : -INFINITY;
  float M = my_lse;
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(grp, M, o, kLanes));
  const float my_w = (M == -INFINITY || my_lse == -INFINITY) ? 0.f : exp2f(my_lse - M);
  float W = my_w;
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) W += __shfl_xor_sync(grp, W, o, kLanes);

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int p = 0; p < kWarpRowMaxParts; ++p) {
    const float wp = __shfl_sync(grp, my_w, p, kLanes);
    if (p < n) {
      const float4 v = po[(size_t)p * kLanes + c];
      acc.x += wp * v.x;
      acc.y += wp * v.y;
      acc.z += wp * v.z;
      acc.w += wp * v.w;
    }
  }
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  if (W > 0.f) {
    res.x = acc.x / W;
    res.y = acc.y / W;
    res.z = acc.z / W;
    res.w = acc.w / W;
  }
  uint2 pk;
  pk.x = E::pack(res.x, res.y);
  pk.y = E::pack(res.z, res.w);
  *reinterpret_cast<uint2*>(out + (size_t)row * D + c * 4) = pk;
}

// Rows with more than kWarpRowMaxParts partitions (long contexts): one CTA per
// row at a time, `ncta` CTAs striding over the rows (rows with fewer
// partitions are skipped). Phase 1 puts the weights of all partitions in
// shared memory (s_w, max_parts floats); phase 2 has every warp (half-warp at
// D = 64) stream an interleaved subset of the partials; a fixed-order merge
// of the streams ends it.
template <typename T, int D>
__device__ __forceinline__ void reduce_rows_split(T* __restrict__ out,
                                                  const float* __restrict__ part_o,
                                                  const float* __restrict__ part_lse,
                                                  const int32_t* __restrict__ context_lens,
                                                  const int32_t* __restrict__ q_start,
                                                  int num_seqs, int num_rows, int num_q_heads,
                                                  int max_context_len, int part_tokens,
                                                  int max_parts, int cta, int ncta, float* s_w) {
  constexpr int kThreadsR = kReduceWarps * 32;
  constexpr int kLanes = D / 4;
  constexpr int kStreams = kThreadsR / kLanes;
  using E = Elem<T>;
  __shared__ float s_red[kThreadsR];
  __shared__ float4 s_acc[kStreams][kLanes];
  const int tid = threadIdx.x;
  for (int row = cta; row < num_rows; row += ncta) {
    int L = context_lens[seq_of_row(row, num_q_heads, q_start, num_seqs)];
    L = L < 0 ? 0 : (L > max_context_len ? max_context_len : L);
    const int n = (L + part_tokens - 1) / part_tokens;
    if (n <= kWarpRowMaxParts) continue;  // uniform over the CTA
    const float* lse = part_lse + (size_t)row * max_parts;
    const float4* po = reinterpret_cast<const float4*>(part_o + (size_t)row * max_parts * D);

    // phase 1: M = max lse (fixed tree), weights, W = sum of weights (fixed tree)
    float m = -INFINITY;
    for (int p = tid; p < n; p += kThreadsR) {
      const float l = lse[p];
      s_w[p] = l;
      m = fmaxf(m, l);
    }
    s_red[tid] = m;
    __syncthreads();
    for (int o = kThreadsR / 2; o > 0; o >>= 1) {
      if (tid < o) s_red[tid] = fmaxf(s_red[tid], s_red[tid + o]);
      __syncthreads();
    }
    const float M = s_red[0];
    __syncthreads();
    float w = 0.f;
    for (int p = tid; p < n; p += kThreadsR) {
      const float l = s_w[p];
      const float e = (M == -INFINITY || l == -INFINITY) ? 0.f : exp2f(l - M);
      s_w[p] = e;
      w += e;
    }
    s_red[tid] = w;
    __syncthreads();
    for (int o = kThreadsR / 2; o > 0; o >>= 1) {
      if (tid < o) s_red[tid] += s_red[tid + o];
      __syncthreads();
    }
    const float W = s_red[0];

    // phase 2: independent weighted loads, one stream per warp (half-warp)
    const int stream = tid / kLanes, c = tid % kLanes;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  #pragma unroll 8
    for (int p = stream; p < n; p += kStreams) {
      const float wp = s_w[p];
      const float4 v = po[(size_t)p * kLanes + c];
      acc.x += wp * v.x;
      acc.y += wp * v.y;
      acc.z += wp * v.z;
      acc.w += wp * v.w;
    }
    s_acc[stream][c] = acc;
    __syncthreads();
    if (tid < kLanes) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  #pragma unroll
      for (int i = 0; i < kStreams; ++i) {
        const float4 v = s_acc[i][tid];
        a.x += v.x;
        a.y += v.y;
        a.z += v.z;
        a.w += v.w;
      }
      float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
      if (W > 0.f) {
        res.x = a.x / W;
        res.y = a.y / W;
        res.z = a.z / W;
        res.w = a.w / W;
      }
      uint2 pk;
      pk.x = E::pack(res.x, res.y);
      pk.y = E::pack(res.z, res.w);
      *reinterpret_cast<uint2*>(out + (size_t)row * D + tid * 4) = pk;
    }
    __syncthreads();  // s_w, s_red and s_acc are reused by the next row
  }
}

// The reduce when no row can have more than kWarpRowMaxParts partitions.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
    lse_reduce_warp_kernel(T* __restrict__ out, const float* __restrict__ part_o,
                           const float* __restrict__ part_lse,
                           const int32_t* __restrict__ context_lens,
                           const int32_t* __restrict__ q_start, int num_seqs, int num_rows,
                           int num_q_heads, int max_context_len, int part_tokens, int max_parts) {
  griddep_wait();  // the partials are complete
  reduce_rows_warp<T, D>(out, part_o, part_lse, context_lens, q_start, num_seqs, num_rows,
                         num_q_heads, max_context_len, part_tokens, max_parts, blockIdx.x);
}

// The reduce otherwise, in one launch: CTAs [0, split_ctas) stride over the
// rows of more than kWarpRowMaxParts partitions (dispatched first: those rows
// are the long pole), the others take the rows of up to kWarpRowMaxParts.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
    lse_reduce_kernel(T* __restrict__ out, const float* __restrict__ part_o,
                      const float* __restrict__ part_lse, const int32_t* __restrict__ context_lens,
                      const int32_t* __restrict__ q_start, int num_seqs, int num_rows,
                      int num_q_heads, int max_context_len, int part_tokens, int max_parts,
                      int split_ctas) {
  extern __shared__ float s_w[];  // [max_parts] weights (split CTAs only)
  griddep_wait();  // the partials are complete
  if ((int)blockIdx.x < split_ctas)
    reduce_rows_split<T, D>(out, part_o, part_lse, context_lens, q_start, num_seqs, num_rows,
                            num_q_heads, max_context_len, part_tokens, max_parts, blockIdx.x,
                            split_ctas, s_w);
  else
    reduce_rows_warp<T, D>(out, part_o, part_lse, context_lens, q_start, num_seqs, num_rows,
                           num_q_heads, max_context_len, part_tokens, max_parts,
                           blockIdx.x - split_ctas);
}

template <typename T, int D>
static cudaError_t launch_reduce_typed(const DecodeLaunch& a, cudaStream_t stream);

// Launch with programmatic stream serialization (the kernel itself waits for
// its predecessor with griddep_wait before reading global memory).
template <typename... Params, typename... Args>
static cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename T, int D, bool kTwoRows, bool kMulti>
static cudaError_t launch_typed(const DecodeLaunch& a, cudaStream_t stream) {
  using SM = DecodeSmem<D>;
  auto kern = decode_partition_kernel<T, D, kTwoRows, kMulti>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc);
  if (e != cudaSuccess) return e;
  // first_part (decode only) > 0: partitions from first_part on
  const int64_t parts = (int64_t)a.max_parts - (kMulti ? 0 : a.first_part);
  dim3 grid((unsigned)(parts * a.max_qtiles), a.num_kv_heads, a.num_seqs);
  e = launch_pdl(kern, grid, dim3(kThreads), SM::kAlloc, stream, a.tm_k, a.tm_v,
                 static_cast<T*>(a.out), a.part_o, a.part_lse, static_cast<const T*>(a.q),
                 a.q_start, a.num_q_tokens, a.max_query_len, a.block_tables, a.bt_stride,
                 a.context_lens, a.num_q_heads, a.group, a.num_blocks, a.max_context_len,
                 a.scale_log2, a.part_blocks, a.max_parts, a.dev_error,
                 kMulti ? 0 : a.first_part);
  if (e != cudaSuccess) return e;
  if (!kMulti && a.first_part > 0 && a.shared_tm_q) {
    // the shared prefix's partitions, overlapping this kernel's end; the
    // reduce after them waits for both
    e = launch_prefill_tc_shared(a, *a.shared_tm_q, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_reduce_typed<T, D>(a, stream);
}

template <typename T, int D>
static cudaError_t launch_reduce_typed(const DecodeLaunch& a, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  if (a.max_parts <= 1) return e;
  const int rows = a.num_q_tokens * a.num_q_heads;
  // Rows of up to kWarpRowMaxParts partitions: a warp (half-warp) each.
  const int rows_per_cta = kReduceWarps * (32 / (D / 4));
  const int warp_ctas = (rows + rows_per_cta - 1) / rows_per_cta;
  if (a.max_parts <= kWarpRowMaxParts) {
    return launch_pdl(lse_reduce_warp_kernel<T, D>, dim3(warp_ctas), dim3(kReduceWarps * 32), 0,
                      stream, static_cast<T*>(a.out), a.part_o, a.part_lse, a.context_lens,
                      a.q_start, a.num_seqs, rows, a.num_q_heads, a.max_context_len,
                      a.part_tokens, a.max_parts);
  }
  // Rows of more: a CTA each, one wave of CTAs striding over the rows.
  auto kern = lse_reduce_kernel<T, D>;
  const size_t wbytes = (size_t)a.max_parts * sizeof(float);
  if (wbytes > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wbytes);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kReduceWarps * 32, wbytes);
  if (e != cudaSuccess) return e;
  const int64_t wave = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  const int split_ctas = (int)(rows < wave ? rows : wave);
  return launch_pdl(kern, dim3(warp_ctas + split_ctas), dim3(kReduceWarps * 32), wbytes, stream,
                    static_cast<T*>(a.out), a.part_o, a.part_lse, a.context_lens, a.q_start,
                    a.num_seqs, rows, a.num_q_heads, a.max_context_len, a.part_tokens,
                    a.max_parts, split_ctas);
}

template <typename T>
static cudaError_t launch_dtype(const DecodeLaunch& a, cudaStream_t stream) {
  if (a.q_start) {  // query chunks: tiles mix tokens and heads, both row halves in use
    return a.head_dim == 128 ? launch_typed<T, 128, true, true>(a, stream)
                             : launch_typed<T, 64, true, true>(a, stream);
  }
  const bool two = a.group > 8;
  if (a.head_dim == 128)
    return two ? launch_typed<T, 128, true, false>(a, stream)
               : launch_typed<T, 128, false, false>(a, stream);
  return two ? launch_typed<T, 64, true, false>(a, stream)
             : launch_typed<T, 64, false, false>(a, stream);
}

cudaError_t launch_reduce(const DecodeLaunch& a, cudaStream_t stream) {
  if (a.bf16)
    return a.head_dim == 128 ? launch_reduce_typed<__nv_bfloat16, 128>(a, stream)
                             : launch_reduce_typed<__nv_bfloat16, 64>(a, stream);
  return a.head_dim == 128 ? launch_reduce_typed<__half, 128>(a, stream)
                           : launch_reduce_typed<__half, 64>(a, stream);
}

template <typename T, int D, bool kTwoRows>
static cudaError_t launch_persistent_typed(const DecodeLaunch& a, cudaStream_t stream) {
  using SM = DecodeSmem<D>;
  auto kern = decode_persistent_kernel<T, D, kTwoRows>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc);
  if (e != cudaSuccess) return e;
  int per_sm = 0;  // resident CTAs per SM, asked per call (cheap next to the launch)
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, SM::kAlloc);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int64_t work_max = (int64_t)a.num_seqs * a.max_parts * a.num_kv_heads;
  const int grid = (int)(work_max < (int64_t)sms * per_sm ? work_max : (int64_t)sms * per_sm);

  decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(a.context_lens, a.num_seqs,
                                                     a.max_context_len, a.part_blocks, a.items,
                                                     a.plan);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the decode grid's prologue (barrier set-up,
  // descriptor prefetch) overlaps the plan; griddepcontrol.wait orders the rest.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SM::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a.tm_k, a.tm_v, static_cast<T*>(a.out), a.part_o,
                         a.part_lse, static_cast<const T*>(a.q), a.block_tables, a.bt_stride,
                         a.context_lens, a.num_seqs, a.num_q_heads, a.group, a.num_kv_heads,
                         a.num_blocks, a.max_context_len, a.scale_log2, a.part_blocks,
                         a.max_parts, static_cast<const uint32_t*>(a.items), a.plan,
                         a.dev_error);
  if (e != cudaSuccess) return e;
  return launch_reduce_typed<T, D>(a, stream);
}

template <typename T>
static cudaError_t launch_persistent_dtype(const DecodeLaunch& a, cudaStream_t stream) {
  const bool two = a.group > 8;
  if (a.head_dim == 128)
    return two ? launch_persistent_typed<T, 128, true>(a, stream)
               : launch_persistent_typed<T, 128, false>(a, stream);
  return two ? launch_persistent_typed<T, 64, true>(a, stream)
             : launch_persistent_typed<T, 64, false>(a, stream);
}

cudaError_t launch_decode_persistent(const DecodeLaunch& a, cudaStream_t stream) {
  return a.bf16 ? launch_persistent_dtype<__nv_bfloat16>(a, stream)
                : launch_persistent_dtype<__half>(a, stream);
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream) {
  return a.bf16 ? launch_dtype<__nv_bfloat16>(a, stream) : launch_dtype<__half>(a, stream);
}

}  // namespace pa
