// pa_cache_ops.cu -- the kernels that keep the paged KV cache current.
//
//  * write_kv: every decode step stores the new token's K and V rows, for
//    every KV head, in the cache slot its sequence's block table gives
//    ("Optimizing LLM Inference: From PagedAttention to AI Infra",
//    "Understanding KV Cache ..."). One CTA per token; each thread moves
//    16-byte vectors, so a row of D = 128 bf16 values is 16 coalesced vectors.
//  * block copies: the copy-on-write fork of a shared block (same page,
//    "Copy-on-Write"; "PagedAttention", "KV Cache Sharing (Copy-on-Write)")
//    and the swap of blocks between GPU memory and CPU RAM for preemption
//    ("PagedAttention", "Managing Virtual Memory (Block Manager)"; "The
//    Memory Wall ...", "The Block Manager"): the whole physical block --
//    every KV head, every slot -- of K and of V, in every layer. Blocks are
//    contiguous, so this is a plain 16-byte-vector copy with several vectors
//    in flight per thread; a pinned host pool is read or written in place
//    over the host link.
#include "pa.h"
#include "pa_internal.h"

namespace pa {

__global__ void __launch_bounds__(256)
    write_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                    uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                    const int64_t* __restrict__ slot_mapping, int num_kv_heads, int vec_per_row,
                    int64_t num_slots, int32_t* __restrict__ dev_error) {
  const int t = blockIdx.x;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (threadIdx.x == 0 && dev_error) atomicAdd(dev_error, 1);
    return;
  }
  const int64_t block = slot / PA_BLOCK_SIZE, offset = slot % PA_BLOCK_SIZE;
  const int n = num_kv_heads * vec_per_row;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int h = i / vec_per_row, c = i - h * vec_per_row;
    const size_t src = ((size_t)t * num_kv_heads + h) * vec_per_row + c;
    const size_t dst = (((size_t)block * num_kv_heads + h) * PA_BLOCK_SIZE + offset) * vec_per_row + c;
    const uint4 kv = __ldg(k + src);
    const uint4 vv = __ldg(v + src);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// Per-layer source and destination pools of a block copy. For copy-on-write
// both sides are the same device pool; for a swap one side is a pinned host
// pool reached through unified addressing.
struct PoolPtrs {
  const uint4* src_k[PA_MAX_LAYERS];
  const uint4* src_v[PA_MAX_LAYERS];
  uint4* dst_k[PA_MAX_LAYERS];
  uint4* dst_v[PA_MAX_LAYERS];
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// One CTA per (pair, layer, K or V): copies one whole block, 16-byte vectors,
// kCopyUnroll of them in flight per thread.
__global__ void __launch_bounds__(kCopyThreads)
    block_copy_kernel(const __grid_constant__ PoolPtrs ptrs,
                      const int64_t* __restrict__ block_mapping, int64_t vec_per_block,
                      int64_t src_num_blocks, int64_t dst_num_blocks,
                      int32_t* __restrict__ dev_error) {
  const int pair = blockIdx.x, layer = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
    if (threadIdx.x == 0 && layer == 0 && !is_v && dev_error) atomicAdd(dev_error, 1);
    return;
  }
  const uint4* s = (is_v ? ptrs.src_v[layer] : ptrs.src_k[layer]) + src * vec_per_block;
  uint4* d = (is_v ? ptrs.dst_v[layer] : ptrs.dst_k[layer]) + dst * vec_per_block;
  int64_t i = threadIdx.x;
  for (; i + (kCopyUnroll - 1) * kCopyThreads < vec_per_block; i += kCopyUnroll * kCopyThreads) {
    uint4 r[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) r[u] = s[i + u * kCopyThreads];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) d[i + u * kCopyThreads] = r[u];
  }
  for (; i < vec_per_block; i += kCopyThreads) d[i] = s[i];
}

cudaError_t launch_write_kv(const void* k, const void* v, void* k_cache, void* v_cache,
                            const int64_t* slot_mapping, int32_t num_tokens,
                            int32_t num_kv_heads, int32_t head_dim, int64_t num_blocks,
                            int32_t* dev_error, cudaStream_t stream) {
  const int vec_per_row = head_dim / 8;
  const int n = num_kv_heads * vec_per_row;
  int threads = ((n + 31) / 32) * 32;
  if (threads > 256) threads = 256;
  write_kv_kernel<<<num_tokens, threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_kv_heads, vec_per_row,
      num_blocks * PA_BLOCK_SIZE, dev_error);
  return cudaGetLastError();
}

cudaError_t launch_block_copy(void* const* src_k, void* const* src_v, void* const* dst_k,
                              void* const* dst_v, int32_t num_layers,
                              const int64_t* block_mapping, int32_t num_pairs,
                              int64_t block_bytes, int64_t src_num_blocks,
                              int64_t dst_num_blocks, int32_t* dev_error, cudaStream_t stream) {
  PoolPtrs ptrs;
  for (int l = 0; l < PA_MAX_LAYERS; ++l) {
    const bool in = l < num_layers;
    ptrs.src_k[l] = in ? static_cast<const uint4*>(src_k[l]) : nullptr;
    ptrs.src_v[l] = in ? static_cast<const uint4*>(src_v[l]) : nullptr;
    ptrs.dst_k[l] = in ? static_cast<uint4*>(dst_k[l]) : nullptr;
    ptrs.dst_v[l] = in ? static_cast<uint4*>(dst_v[l]) : nullptr;
  }
  dim3 grid(num_pairs, num_layers, 2);
  block_copy_kernel<<<grid, kCopyThreads, 0, stream>>>(ptrs, block_mapping, block_bytes / 16,
                                                       src_num_blocks, dst_num_blocks, dev_error);
  return cudaGetLastError();
}

}  // namespace pa
