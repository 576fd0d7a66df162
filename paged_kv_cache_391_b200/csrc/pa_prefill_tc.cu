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
// One CTA per (128-row query tile, partition, KV head, sequence); tile rows are
// (query token, head) pairs of the KV head's query group. 160 threads:
//  * warps 0-3: softmax. Thread r owns row r: TMEM lane r of S and O.
//  * warp 4, one lane: producer. It issues every TMA load (Q once; per step
//    K and V of 4 cache blocks = 64 keys into a 2-stage ring) and every MMA:
//      S[j%2] = Q K_j^T        (M=128, N=64, K=D; both operands K-major)
//      O     += P_j V_j        (M=128, N=D, K=64; P K-major, V MN-major)
//    S is double-buffered in TMEM so S(j+1) runs while the softmax of step j
//    does. P_j (bf16) is written by the softmax warps into the shared memory
//    of K_j, which S(j) no longer needs.
// Online softmax per row in fp32, base 2; O is rescaled in TMEM when a row's
// maximum grows. Keys past the context, past the row's causal limit, or in a
// block with a bad table entry are masked to -inf, and V rows past the context
// are zeroed before P.V (0 * stale data must stay 0). All waits are bounded;
// TMEM is released on every path.
#include <math.h>

#include <type_traits>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;                 // query rows per CTA (M)
constexpr int kKeys = 64;                  // keys per step (4 cache blocks)
constexpr int kStepBlocks = kKeys / 16;
constexpr int kD = 128;                    // head dim of this path
constexpr int kChunks = kD / 64;           // 128-byte swizzle columns of a row
constexpr int kSoftmaxWarps = 4;
constexpr int kThreadsTc = (kSoftmaxWarps + 1) * 32;
constexpr uint32_t kTmemCols = 256;        // S0 [0,64) S1 [64,128) O [128,256)
constexpr uint32_t kOCol = 128;

constexpr int kQBytes = kRows * kD * 2;            // 32 KiB: [chunk][128 rows][128 B]
constexpr int kKBytes = kKeys * kD * 2;            // 16 KiB: [chunk][64 keys][128 B]; later P
constexpr int kVBytes = kKeys * kD * 2;            // 16 KiB: [chunk][64 keys][128 B]
constexpr int kStageBytes = kKBytes + kVBytes;
constexpr int kQOff = 0;
constexpr int kStageOff = kQBytes;
constexpr int kBarOff = kStageOff + 2 * kStageBytes;
// barriers: q_full, kv_full[2], s_full[2], p_ready, pv_done ; then the TMEM address
constexpr int kNumBars = 7;
constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
constexpr int kSmemBytes = kTmemSlotOff + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kRows * 128 == kKBytes, "P (128 rows x 64 bf16) must fit in a K stage");

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk16) {
  return row * 128 + ((chunk16 ^ (row & 7)) << 4);
}

template <typename T>
__global__ void __launch_bounds__(kThreadsTc)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, T* __restrict__ out,
                      float* __restrict__ part_o, float* __restrict__ part_lse,
                      const int32_t* __restrict__ q_start, int num_q_tokens, int max_query_len,
                      const int32_t* __restrict__ block_tables, int bt_stride,
                      const int32_t* __restrict__ context_lens, int num_q_heads, int group,
                      int64_t num_blocks, int max_context_len, float scale_log2,
                      int part_blocks, int max_parts, int32_t* __restrict__ dev_error) {
  using E = Elem<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;  // [2]
  uint64_t* s_full = bars + 3;   // [2]
  uint64_t* p_ready = bars + 5;
  uint64_t* pv_done = bars + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemSlotOff);

  const int kvh = blockIdx.y, seq = blockIdx.z;
  const int part = (int)(blockIdx.x % (unsigned)max_parts);
  const int qtile = (int)(blockIdx.x / (unsigned)max_parts);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool counter = part == 0 && kvh == 0 && qtile == 0 && tid == 0 && dev_error;

  // ---- the CTA's rows and keys (uniform over the CTA; exits before any barrier)
  int L = context_lens[seq];
  if (L < 0 || L > max_context_len) {
    if (counter) atomicAdd(dev_error, 1);
    L = L < 0 ? 0 : max_context_len;
  }
  const int q0 = q_start[seq];
  int Tq = q_start[seq + 1] - q0;
  if (q0 < 0 || Tq < 0 || q0 + Tq > num_q_tokens) {
    if (counter) atomicAdd(dev_error, 1);
    return;
  }
  if (Tq > min(L, max_query_len)) {
    if (counter) atomicAdd(dev_error, 1);
    Tq = min(L, max_query_len);
  }
  const int tok_per_tile = kRows / group;
  const int t0 = qtile * tok_per_tile;
  if (t0 >= Tq) return;
  const int nblk_seq = (L + 15) / 16;
  const int n_parts = nblk_seq > 0 ? (nblk_seq + part_blocks - 1) / part_blocks : 1;
  if (part >= n_parts) return;
  const int key_begin = part * part_blocks * 16;
  const int t_last = min(t0 + tok_per_tile, Tq) - 1;
  // keys this tile can see in this partition: up to the last row's causal limit
  const int key_end = min(min((part + 1) * part_blocks * 16, L), L - Tq + t_last + 1);
  const int n_steps = key_end > key_begin ? (key_end - key_begin + kKeys - 1) / kKeys : 0;
  const int q_head0 = kvh * group;

  // ---- set-up: barriers (thread 0), TMEM (warp 0)
  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_ready, kSoftmaxWarps * 32);
    mbar_init(pv_done, 1);
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

  const uint32_t q_s = smem_addr(smem + kQOff);
  auto stage_k = [&](int st) { return smem + kStageOff + st * kStageBytes; };
  auto stage_v = [&](int st) { return smem + kStageOff + st * kStageBytes + kKBytes; };
  const int32_t* bt_row = block_tables + (size_t)seq * bt_stride;

  if (warp == kSoftmaxWarps) {
    // =============================== producer ===============================
    if (lane == 0) {
      const uint32_t id_s = tc::instr_desc_f16(Elem<T>::kBf16, kRows, kKeys, false, false);
      const uint32_t id_pv = tc::instr_desc_f16(Elem<T>::kBf16, kRows, kD, false, true);
      // What is in flight, for the drain after a wait that gave up.
      int kv_pending[2] = {-1, -1};     // step whose K/V load into the stage is unconfirmed
      uint64_t* last_bar = nullptr;     // barrier of the last MMA commit, and its parity
      uint32_t last_parity = 0;
      auto load_kv = [&](int j) {
        const int st = j & 1;
        kv_pending[st] = j;
        uint32_t bytes = 0;
        const int lb0 = key_begin / 16 + j * kStepBlocks;
        int pids[kStepBlocks];
#pragma unroll
        for (int b = 0; b < kStepBlocks; ++b) {
          const int lb = lb0 + b;
          int p = -1;
          if (lb * 16 < key_end) {
            p = __ldg(bt_row + lb);
            if (p < 0 || p >= num_blocks) p = -1;
          }
          pids[b] = p;
          if (p >= 0) bytes += 2 * kChunks * 2048;
        }
        if (bytes == 0) {
          mbar_arrive(&kv_full[st]);
          return;
        }
        mbar_arrive_expect_tx(&kv_full[st], bytes);
#pragma unroll
        for (int b = 0; b < kStepBlocks; ++b) {
          if (pids[b] < 0) continue;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            tma_load_4d(stage_k(st) + c * (kKeys * 128) + b * 2048, &tm_k, &kv_full[st], c * 64,
                        0, kvh, pids[b]);
            tma_load_4d(stage_v(st) + c * (kKeys * 128) + b * 2048, &tm_v, &kv_full[st], c * 64,
                        0, kvh, pids[b]);
          }
        }
      };
      auto issue_s = [&](int j) {
        const int st = j & 1;
        const uint32_t k_s = smem_addr(stage_k(st));
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 columns = 32 bytes into the swizzled row
          const uint64_t a = tc::smem_desc_sw128(q_s + (kk >> 2) * (kRows * 128) + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(k_s + (kk >> 2) * (kKeys * 128) + off, 16, 1024);
          tc::mma_f16(tmem + (uint32_t)(st * kKeys), a, b, id_s, kk > 0);
        }
        tc::commit(&s_full[st]);
        last_bar = &s_full[st];
        last_parity = (uint32_t)((j >> 1) & 1);
      };
      auto issue_pv = [&](int j) {
        const int st = j & 1;
        const uint32_t p_s = smem_addr(stage_k(st));
        const uint32_t v_s = smem_addr(stage_v(st));
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t a = tc::smem_desc_sw128(p_s + kk * 32, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(v_s + kk * 2048, kKeys * 128, 1024);
          tc::mma_f16(tmem + kOCol, a, b, id_pv, j > 0 || kk > 0);
        }
        tc::commit(pv_done);
        last_bar = pv_done;
        last_parity = (uint32_t)(j & 1);
      };
      auto wait_kv = [&](int j) {
        const bool ok = mbar_wait(&kv_full[j & 1], (j >> 1) & 1);
        if (ok) kv_pending[j & 1] = -1;
        return ok;
      };

      tma_prefetch_desc(&tm_q);
      if (n_steps > 0) {
        mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          tc::tma_load_3d(smem + kQOff + c * (kRows * 128), &tm_q, q_full, c * 64, q_head0,
                          q0 + t0);
        load_kv(0);
        if (n_steps > 1) load_kv(1);
        failed = !mbar_wait(q_full, 0) || !wait_kv(0);
        if (!failed) {
          tc::fence_after_sync();
          issue_s(0);
        }
      }
      for (int j = 0; j < n_steps && !failed; ++j) {
        if (j + 1 < n_steps) {
          if (!wait_kv(j + 1)) { failed = true; break; }
          issue_s(j + 1);
        }
        if (!mbar_wait(p_ready, j & 1)) { failed = true; break; }
        tc::fence_after_sync();
        issue_pv(j);
        if (j + 2 < n_steps) {
          if (!mbar_wait(pv_done, j & 1)) { failed = true; break; }
          load_kv(j + 2);
        }
      }
      if (failed) {
        // Let the copies and MMAs already issued finish (each wait bounded)
        // before shared memory and TMEM are released.
        (void)mbar_wait(q_full, 0);
        for (int st = 0; st < 2; ++st)
          if (kv_pending[st] >= 0) (void)mbar_wait(&kv_full[st], (kv_pending[st] >> 1) & 1);
        if (last_bar) (void)mbar_wait(last_bar, last_parity);
        if (dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
      }
    }
  } else {
    // =============================== softmax ================================
    const int r = tid;                                   // tile row = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const int t = t0 + r / group, h = r % group;         // query token in the chunk, head
    const bool row_ok = t < Tq;
    const int lim = L - Tq + (row_ok ? t : 0);           // last key this row may see
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < n_steps; ++j) {
      const int st = j & 1;
      const int kb = key_begin + j * kKeys;
      // table entries of this step (validity only)
      int bad_mask = 0;
#pragma unroll
      for (int b = 0; b < kStepBlocks; ++b) {
        const int lb = kb / 16 + b;
        if (lb * 16 < key_end) {
          const int p = __ldg(bt_row + lb);
          if (p < 0 || p >= num_blocks) bad_mask |= 1 << b;
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1))) { failed = true; break; }
      tc::fence_after_sync();
      float s[64];
      {
        float a[32], b2[32];
        tc::tmem_ld32(lane_addr + (uint32_t)(st * kKeys), a);
        tc::tmem_ld32(lane_addr + (uint32_t)(st * kKeys + 32), b2);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = a[i];
          s[32 + i] = b2[i];
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const int kp = kb + i;
        const bool ok = kp < key_end && kp <= lim && !((bad_mask >> (i >> 4)) & 1);
        s[i] = ok ? s[i] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float m_new = fmaxf(m, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = exp2f(m - m_use);
      uint32_t pk[32];
      float psum = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        pk[i] = E::pack(exp2f(s[2 * i] - m_use), exp2f(s[2 * i + 1] - m_use));
        const float2 u = E::unpack(pk[i]);
        psum += u.x + u.y;
      }
      l = l * alpha + psum;
      m = m_new;
      // PV(j-1) must be done: it read the P buffer this step reuses' twin and
      // writes O, which may be rescaled below.
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1))) { failed = true; break; }
      tc::fence_after_sync();
      // P row r: 64 bf16 = 128 bytes, 128-byte swizzle, in K_j's shared memory
      uint8_t* p_row = stage_k(st);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(p_row + swz(r, c)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      // V rows of keys past the context (the final step only) become zero
      if (kb + kKeys > key_end || bad_mask) {
        uint8_t* v = stage_v(st);
        for (int i = r; i < kKeys * kChunks * 8; i += kSoftmaxWarps * 32) {
          const int c = i / (kKeys * 8), rem = i % (kKeys * 8);
          const int key = rem / 8;
          if (kb + key >= key_end || ((bad_mask >> (key >> 4)) & 1))
            *reinterpret_cast<uint4*>(v + c * (kKeys * 128) + key * 128 + (rem % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // rescale O when this row's maximum grew (warp-uniform decision)
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          float o[32];
          tc::tmem_ld32(lane_addr + kOCol + c * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tc::tmem_st32(lane_addr + kOCol + c * 32, o);
        }
        tc::tmem_wait_st();
      }
      fence_proxy_async_smem();   // P and zeroed V rows -> visible to the tensor core
      tc::fence_before_sync();
      mbar_arrive(p_ready);
    }
    // ---- epilogue: O / l  ->  out (one partition) or fp32 partials
    if (!failed && n_steps > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(pv_done, (n_steps - 1) & 1)))
      failed = true;
    if (failed) {
      if (lane == 0 && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
    } else {
      tc::fence_after_sync();
      const bool direct = n_parts == 1;
      const size_t orow = (size_t)(q0 + t) * num_q_heads + q_head0 + h;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        float o[32];
        if (n_steps > 0) {
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
            float4* dst = reinterpret_cast<float4*>(part_o + (orow * max_parts + part) * kD + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(o[4 * v] * inv, o[4 * v + 1] * inv, o[4 * v + 2] * inv,
                                   o[4 * v + 3] * inv);
          }
        }
      }
      if (row_ok && !direct)
        part_lse[orow * max_parts + part] = l > 0.f ? m + log2f(l) : -INFINITY;
    }
  }

  // ---- teardown: every thread done with TMEM, then warp 0 frees it
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

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
    dim3 grid((unsigned)((int64_t)a.max_parts * qtiles), a.num_kv_heads, a.num_seqs);
    kern<<<grid, kThreadsTc, kSmemAlloc, stream>>>(
        tm_q, a.tm_k, a.tm_v, static_cast<T*>(a.out), a.part_o, a.part_lse, a.q_start,
        a.num_q_tokens, a.max_query_len, a.block_tables, a.bt_stride, a.context_lens,
        a.num_q_heads, a.group, a.num_blocks, a.max_context_len, a.scale_log2, a.part_blocks,
        a.max_parts, a.dev_error);
    return cudaGetLastError();
  };
  return a.bf16 ? run((__nv_bfloat16*)nullptr) : run((__half*)nullptr);
}

}  // namespace pa
