// pa_cache_ops.cu -- the kernels that keep the paged KV cache current.
//
//  * write_kv: every decode step stores the new token's K and V rows, for
//    every KV head, in the cache slot its sequence's block table gives
//    ("Optimizing LLM Inference: From PagedAttention to AI Infra",
//    "Understanding KV Cache ..."). One CTA per token; each thread moves
//    16-byte vectors, so a row of D = 128 bf16 values is 16 coalesced vectors.
//  * copy_blocks: the copy-on-write fork of a shared block (same page,
//    "Copy-on-Write"; "PagedAttention", "KV Cache Sharing (Copy-on-Write)"):
//    the whole physical block -- every KV head, every slot -- of K and of V,
//    in every layer. Blocks are contiguous in HBM, so this is a plain
//    16-byte-vector copy with several vectors in flight per thread.
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

struct LayerPtrs {
  uint4* k[PA_MAX_LAYERS];
  uint4* v[PA_MAX_LAYERS];
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(const __grid_constant__ LayerPtrs ptrs,
                       const int64_t* __restrict__ block_mapping, int64_t vec_per_block,
                       int64_t num_blocks, int32_t* __restrict__ dev_error) {
  const int pair = blockIdx.x, layer = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && layer == 0 && !is_v && dev_error) atomicAdd(dev_error, 1);
    return;
  }
  uint4* base = is_v ? ptrs.v[layer] : ptrs.k[layer];
  const uint4* s = base + src * vec_per_block;
  uint4* d = base + dst * vec_per_block;
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

cudaError_t launch_copy_blocks(void* const* k_caches, void* const* v_caches, int32_t num_layers,
                               const int64_t* block_mapping, int32_t num_pairs,
                               int64_t block_bytes, int64_t num_blocks, int32_t* dev_error,
                               cudaStream_t stream) {
  LayerPtrs ptrs;
  for (int l = 0; l < PA_MAX_LAYERS; ++l) {
    ptrs.k[l] = l < num_layers ? static_cast<uint4*>(k_caches[l]) : nullptr;
    ptrs.v[l] = l < num_layers ? static_cast<uint4*>(v_caches[l]) : nullptr;
  }
  dim3 grid(num_pairs, num_layers, 2);
  copy_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(ptrs, block_mapping, block_bytes / 16,
                                                        num_blocks, dev_error);
  return cudaGetLastError();
}

}  // namespace pa
