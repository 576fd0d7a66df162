// pa_api.cu -- libpa's C ABI (declared in include/pa.h): argument checks,
// launch geometry, workspace sizing and TMA descriptor encoding. Allocates
// no device memory and never synchronises the caller's stream.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

pa_status cuda_fail(cudaError_t e) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return PA_ERR_CUDA;
}

pa_status driver_fail(const char* what, int code) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s failed (CUresult %d)", what, code);
  return PA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_dtype(pa_dtype d) { return d == PA_DTYPE_F16 || d == PA_DTYPE_BF16; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The cache pool [NB][H_kv][16][D] as a 4-D tensor (D innermost); a box is
// 64 columns x 16 slots of one (block, KV head), landing as 16 rows of 128
// bytes with the 128-byte swizzle.
pa_status encode_pool_map(CUtensorMap* map, const void* pool, int64_t num_blocks,
                          int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype) {
  auto encode = tensor_map_encoder();
  if (!encode) return driver_fail("cuTensorMapEncodeTiled lookup", -1);
  const cuuint64_t row = (cuuint64_t)head_dim * 2;
  cuuint64_t dims[4] = {(cuuint64_t)head_dim, PA_BLOCK_SIZE, (cuuint64_t)num_kv_heads,
                        (cuuint64_t)num_blocks};
  cuuint64_t strides[3] = {row, row * PA_BLOCK_SIZE, row * PA_BLOCK_SIZE * num_kv_heads};
  cuuint32_t box[4] = {64, PA_BLOCK_SIZE, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map,
                      dtype == PA_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                      4, const_cast<void*>(pool), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return driver_fail("cuTensorMapEncodeTiled", (int)r);
  return PA_OK;
}

// q [tokens][H_q][D] as a 3-D tensor (D innermost); a box is 64 columns x the
// `group` heads of one KV head x 128 / group tokens = 128 rows of 128 bytes,
// 128-byte swizzled: one K-major operand chunk of a 128-row query tile.
pa_status encode_query_map(CUtensorMap* map, const void* q, int32_t num_q_tokens,
                           int32_t num_q_heads, int32_t head_dim, int32_t group, pa_dtype dtype) {
  auto encode = tensor_map_encoder();
  if (!encode) return driver_fail("cuTensorMapEncodeTiled lookup", -1);
  const cuuint64_t row = (cuuint64_t)head_dim * 2;
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)num_q_tokens};
  cuuint64_t strides[2] = {row, row * num_q_heads};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(128 / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map,
                      dtype == PA_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                      3, const_cast<void*>(q), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return driver_fail("cuTensorMapEncodeTiled (query)", (int)r);
  return PA_OK;
}

int64_t max_partitions(int32_t max_context_len, int32_t partition_tokens) {
  if (partition_tokens <= 0 || max_context_len <= partition_tokens) return 1;
  return ((int64_t)max_context_len + partition_tokens - 1) / partition_tokens;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

namespace pa {
pa_status record_cuda_error(cudaError_t e) { return cuda_fail(e); }

pa_status device_view(const void* p, void** dev_ptr) {
  if (!p) return PA_ERR_INVALID_ARG;
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // do not leave this error for a later call to report
    return PA_ERR_INVALID_ARG;
  }
  switch (attr.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      *dev_ptr = const_cast<void*>(p);
      return PA_OK;
    case cudaMemoryTypeHost:
      if (!attr.devicePointer) return PA_ERR_INVALID_ARG;
      *dev_ptr = attr.devicePointer;
      return PA_OK;
    default:
      return PA_ERR_INVALID_ARG;  // pageable host memory: not reachable from kernels
  }
}
}  // namespace pa

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case PA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_OUT_OF_BLOCKS: return "out of KV cache blocks";
  }
  return "unknown status";
}

const char* pa_last_cuda_error(void) { return g_last_cuda_error; }

pa_status pa_write_kv(const void* k, const void* v, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                      int32_t* dev_error, void* stream) {
  if (num_tokens < 0 || num_kv_heads < 1 || num_blocks < 1 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (block_size != PA_BLOCK_SIZE || head_dim < 8 || head_dim > 1024 || head_dim % 8)
    return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8) || (dev_error && !aligned(dev_error, 4)))
    return PA_ERR_INVALID_ARG;
  cudaError_t e = pa::launch_write_kv(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                      num_kv_heads, head_dim, num_blocks, dev_error,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const int64_t parts = max_partitions(max_context_len, partition_tokens);
  if (parts <= 1) return 0;
  const size_t rows = (size_t)num_seqs * num_q_heads * parts;
  return round256(rows * head_dim * sizeof(float)) + round256(rows * sizeof(float));
}

size_t pa_decode_persistent_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                           int32_t head_dim, int32_t max_context_len,
                                           int32_t partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const int64_t parts = max_partitions(max_context_len, partition_tokens);
  return pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                  partition_tokens) +
         round256((size_t)num_seqs * parts * sizeof(uint32_t)) + 256;
}

// The chunk path's plan (longest-first order of the tcgen05 kernel's work):
// item list and counter after the partials, or 0 when the tcgen05 path does
// not apply.
size_t chunk_plan_bytes(int32_t num_seqs, int32_t group_size, int32_t head_dim,
                        int32_t max_query_len, int64_t parts, int32_t partition_tokens) {
  if (num_seqs <= 0 || group_size <= 0 ||
      !pa::prefill_tc_eligible(head_dim, group_size, max_query_len, parts, partition_tokens))
    return 0;
  const int64_t items = pa::prefill_tc_max_items(num_seqs, max_query_len, group_size, parts);
  return round256((size_t)items * 8) + 256;
}

size_t pa_prefill_chunk_workspace_size(int32_t num_q_tokens, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t group_size, int32_t head_dim,
                                       int32_t max_query_len, int32_t max_context_len,
                                       int32_t partition_tokens) {
  if (num_q_tokens <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  return pa_decode_workspace_size(num_q_tokens, num_q_heads, head_dim, max_context_len,
                                  partition_tokens) +
         chunk_plan_bytes(num_seqs, group_size, head_dim, max_query_len,
                          max_partitions(max_context_len, partition_tokens), partition_tokens);
}

}  // extern "C"

namespace {

// The common body of pa_decode (q_start == NULL: one query token per
// sequence) and pa_prefill_chunk (q_start[s] .. q_start[s + 1] are the query
// tokens of sequence s, the last ones of its context).
pa_status attention(void* out, const void* q, const int32_t* q_start, int32_t num_q_tokens,
                    int32_t max_query_len, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t group_size, int32_t head_dim, int32_t block_size,
                    int64_t num_blocks, int32_t max_context_len, float scale,
                    int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                    int32_t* dev_error, pa_dtype dtype, void* stream, bool persistent = false,
                    int32_t shared_tokens = 0) {
  if (num_seqs < 0 || num_q_heads < 1 || group_size < 1 || num_blocks < 1 ||
      max_context_len < 0 || partition_tokens < 0 || !valid_dtype(dtype) || !isfinite(scale) ||
      num_q_tokens < 0 || max_query_len < 0 || shared_tokens < 0 ||
      shared_tokens > max_context_len)
    return PA_ERR_INVALID_ARG;
  if (block_size != PA_BLOCK_SIZE || (head_dim != 64 && head_dim != 128) || group_size > 16 ||
      num_q_heads % group_size != 0 || partition_tokens % PA_BLOCK_SIZE != 0)
    return PA_ERR_UNSUPPORTED;
  const int32_t num_kv_heads = num_q_heads / group_size;
  if (num_seqs > 65535 || num_kv_heads > 65535 || num_blocks > (int64_t(1) << 32) ||
      (int64_t)num_q_tokens * num_q_heads > 0x7fffffff)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_q_tokens == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || (dev_error && !aligned(dev_error, 4)) ||
      (q_start && !aligned(q_start, 4)))
    return PA_ERR_INVALID_ARG;
  const int64_t max_blocks = ((int64_t)max_context_len + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE;
  if (block_table_stride < max_blocks || block_table_stride < 1) return PA_ERR_INVALID_ARG;

  const int64_t parts = max_partitions(max_context_len, partition_tokens);
  const int64_t qtiles = q_start ? ((int64_t)max_query_len * group_size + 15) / 16 : 1;
  if (qtiles < 1) return PA_OK;  // no query token can exist
  if (parts * qtiles > 0x7fffffff) return PA_ERR_UNSUPPORTED;
  // The work queue packs (sequence, partition) into 16 + 16 bits and counts
  // (item, KV head) pairs in 32 bits.
  if (persistent && (parts > 65536 || (int64_t)num_seqs * parts * num_kv_heads > 0x7fffffff))
    return PA_ERR_UNSUPPORTED;
  const size_t need = pa_decode_workspace_size(num_q_tokens, num_q_heads, head_dim,
                                               max_context_len, partition_tokens);
  const size_t need_all =
      persistent ? pa_decode_persistent_workspace_size(num_q_tokens, num_q_heads, head_dim,
                                                       max_context_len, partition_tokens)
                 : need;
  if (need_all > 0) {
    if (!workspace || !aligned(workspace, 256)) return PA_ERR_INVALID_ARG;
    if (workspace_bytes < need_all) return PA_ERR_WORKSPACE_TOO_SMALL;
  }

  pa::DecodeLaunch a;
  pa_status st = encode_pool_map(&a.tm_k, k_cache, num_blocks, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  st = encode_pool_map(&a.tm_v, v_cache, num_blocks, num_kv_heads, head_dim, dtype);
  if (st != PA_OK) return st;
  const size_t rows = (size_t)num_q_tokens * num_q_heads * parts;
  a.out = out;
  a.part_o = need ? static_cast<float*>(workspace) : nullptr;
  a.part_lse = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                               round256(rows * head_dim * sizeof(float)))
                    : nullptr;
  a.q = q;
  a.q_start = q_start;
  a.num_q_tokens = num_q_tokens;
  a.max_query_len = q_start ? max_query_len : 1;
  a.max_qtiles = (int32_t)qtiles;
  a.block_tables = block_tables;
  a.bt_stride = block_table_stride;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group_size;
  a.head_dim = head_dim;
  a.num_blocks = num_blocks;
  a.max_context_len = max_context_len;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);  // scale * log2(e)
  a.part_tokens = parts > 1 ? partition_tokens : (int32_t)(max_blocks * PA_BLOCK_SIZE);
  a.part_blocks = parts > 1 ? partition_tokens / PA_BLOCK_SIZE : (int32_t)(max_blocks > 0 ? max_blocks : 1);
  if (a.part_tokens < PA_BLOCK_SIZE) a.part_tokens = PA_BLOCK_SIZE;
  a.max_parts = (int32_t)parts;
  a.dev_error = dev_error;
  a.bf16 = dtype == PA_DTYPE_BF16;
  a.items = nullptr;
  a.plan = nullptr;
  a.chunk_items = nullptr;
  a.chunk_plan = nullptr;
  a.first_part = 0;
  a.shared_tm_q = nullptr;
  if (persistent) {
    char* tail = static_cast<char*>(workspace) + need;
    a.items = reinterpret_cast<uint32_t*>(tail);
    a.plan = reinterpret_cast<int32_t*>(tail + round256((size_t)num_seqs * parts * sizeof(uint32_t)));
    cudaError_t e = pa::launch_decode_persistent(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_fail(e);
  }
  // Long query chunks (at least 64 rows of (token, head) per KV head) are a
  // dense contraction: run them on the tcgen05 tensor cores.
  if (q_start && (int64_t)max_query_len * group_size >= 64 && pa::prefill_tc_supported(a)) {
    // With room after the partials (pa_prefill_chunk_workspace_size), a plan
    // kernel orders the work longest first; otherwise the grid's order.
    const size_t plan = chunk_plan_bytes(num_seqs, group_size, head_dim, max_query_len, parts,
                                         partition_tokens);
    if (plan && workspace && aligned(workspace, 256) && workspace_bytes >= need + plan &&
        pa::prefill_tc_max_items(num_seqs, max_query_len, group_size, parts) * num_kv_heads <=
            0x7fffffff - 65536) {  // the work counter passes the item count by one per CTA
      char* tail = static_cast<char*>(workspace) + need;
      const int64_t items = pa::prefill_tc_max_items(num_seqs, max_query_len, group_size, parts);
      a.chunk_items = reinterpret_cast<uint2*>(tail);
      a.chunk_plan = reinterpret_cast<int32_t*>(tail + round256((size_t)items * 8));
    }
    CUtensorMap tm_q;
    st = encode_query_map(&tm_q, q, num_q_tokens, num_q_heads, head_dim, group_size, dtype);
    if (st != PA_OK) return st;
    cudaError_t e = pa::launch_prefill_tc(a, tm_q, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = pa::launch_reduce(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_fail(e);
  }
  // A prefix shared by every sequence: its whole partitions (at least two,
  // and not the last one) as one tcgen05 contraction over all sequences'
  // queries, the rest by the decode kernel, the reduce over both.
  if (!q_start && shared_tokens > 0 && parts > 2) {
    const int64_t pp = shared_tokens / a.part_tokens;
    a.first_part = (int32_t)(pp < parts - 1 ? pp : parts - 1);
    if (a.first_part >= 2 && pa::prefill_tc_shared_supported(a)) {
      CUtensorMap tm_q;
      st = encode_query_map(&tm_q, q, num_q_tokens, num_q_heads, head_dim, group_size, dtype);
      if (st != PA_OK) return st;
      a.shared_tm_q = &tm_q;  // the decode's launch runs the prefix kernel after its own
      cudaError_t e = pa::launch_decode(a, static_cast<cudaStream_t>(stream));
      return e == cudaSuccess ? PA_OK : cuda_fail(e);
    }
    a.first_part = 0;
  }
  cudaError_t e = pa::launch_decode(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t group_size, int32_t head_dim, int32_t block_size,
                    int64_t num_blocks, int32_t max_context_len, float scale,
                    int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                    int32_t* dev_error, pa_dtype dtype, void* stream) {
  return attention(out, q, nullptr, num_seqs, 1, k_cache, v_cache, block_tables,
                   block_table_stride, context_lens, num_seqs, num_q_heads, group_size, head_dim,
                   block_size, num_blocks, max_context_len, scale, partition_tokens, workspace,
                   workspace_bytes, dev_error, dtype, stream);
}

pa_status pa_decode_persistent(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               int32_t block_table_stride, const int32_t* context_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                               int32_t head_dim, int32_t block_size, int64_t num_blocks,
                               int32_t max_context_len, float scale, int32_t partition_tokens,
                               void* workspace, size_t workspace_bytes, int32_t* dev_error,
                               pa_dtype dtype, void* stream) {
  return attention(out, q, nullptr, num_seqs, 1, k_cache, v_cache, block_tables,
                   block_table_stride, context_lens, num_seqs, num_q_heads, group_size, head_dim,
                   block_size, num_blocks, max_context_len, scale, partition_tokens, workspace,
                   workspace_bytes, dev_error, dtype, stream, true);
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  int32_t block_table_stride, const int32_t* context_lens,
                                  int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                                  int32_t head_dim, int32_t block_size, int64_t num_blocks,
                                  int32_t max_context_len, float scale,
                                  int32_t shared_prefix_tokens, int32_t partition_tokens,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                  pa_dtype dtype, void* stream) {
  return attention(out, q, nullptr, num_seqs, 1, k_cache, v_cache, block_tables,
                   block_table_stride, context_lens, num_seqs, num_q_heads, group_size, head_dim,
                   block_size, num_blocks, max_context_len, scale, partition_tokens, workspace,
                   workspace_bytes, dev_error, dtype, stream, false, shared_prefix_tokens);
}

pa_status pa_prefill_chunk(void* out, const void* q, const int32_t* q_start,
                           int32_t num_q_tokens, int32_t max_query_len, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           int32_t block_table_stride, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                           int32_t head_dim, int32_t block_size, int64_t num_blocks,
                           int32_t max_context_len, float scale, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, int32_t* dev_error,
                           pa_dtype dtype, void* stream) {
  if (!q_start) return PA_ERR_INVALID_ARG;
  return attention(out, q, q_start, num_q_tokens, max_query_len, k_cache, v_cache, block_tables,
                   block_table_stride, context_lens, num_seqs, num_q_heads, group_size, head_dim,
                   block_size, num_blocks, max_context_len, scale, partition_tokens, workspace,
                   workspace_bytes, dev_error, dtype, stream);
}

pa_status pa_copy_blocks(void* const* k_caches, void* const* v_caches, int32_t num_layers,
                         const int64_t* block_mapping, int32_t num_pairs, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int64_t num_blocks,
                         pa_dtype dtype, int32_t* dev_error, void* stream) {
  if (num_layers < 1 || num_pairs < 0 || num_kv_heads < 1 || num_blocks < 1 ||
      !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_layers > PA_MAX_LAYERS || block_size != PA_BLOCK_SIZE || head_dim < 8 ||
      head_dim % 8)
    return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!k_caches || !v_caches || !block_mapping || !aligned(block_mapping, 8) ||
      (dev_error && !aligned(dev_error, 4)))
    return PA_ERR_INVALID_ARG;
  for (int l = 0; l < num_layers; ++l)
    if (!k_caches[l] || !v_caches[l] || !aligned(k_caches[l], 16) || !aligned(v_caches[l], 16))
      return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = (int64_t)num_kv_heads * PA_BLOCK_SIZE * head_dim * 2;
  cudaError_t e = pa::launch_block_copy(k_caches, v_caches, k_caches, v_caches, num_layers,
                                        block_mapping, num_pairs, block_bytes, num_blocks,
                                        num_blocks, dev_error, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

pa_status pa_swap_blocks(void* const* src_k, void* const* src_v, void* const* dst_k,
                         void* const* dst_v, int32_t num_layers, const int64_t* block_mapping,
                         int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                         int32_t block_size, int64_t src_num_blocks, int64_t dst_num_blocks,
                         pa_dtype dtype, int32_t* dev_error, void* stream) {
  if (num_layers < 1 || num_pairs < 0 || num_kv_heads < 1 || src_num_blocks < 1 ||
      dst_num_blocks < 1 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_layers > PA_MAX_LAYERS || block_size != PA_BLOCK_SIZE || head_dim < 8 ||
      head_dim % 8)
    return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!src_k || !src_v || !dst_k || !dst_v || !block_mapping || !aligned(block_mapping, 8) ||
      (dev_error && !aligned(dev_error, 4)))
    return PA_ERR_INVALID_ARG;
  // Every pool, the mapping and the error counter must be reachable from the
  // device: device memory, managed memory, or pinned / registered host
  // memory (translated to its device address). Pageable host memory is
  // refused here instead of faulting in the kernel.
  void* dk[PA_MAX_LAYERS];
  void* dv[PA_MAX_LAYERS];
  void* sk[PA_MAX_LAYERS];
  void* sv[PA_MAX_LAYERS];
  void* const* in[4] = {src_k, src_v, dst_k, dst_v};
  void** outp[4] = {sk, sv, dk, dv};
  for (int a = 0; a < 4; ++a) {
    for (int l = 0; l < num_layers; ++l) {
      void* dp = nullptr;
      pa_status st = pa::device_view(in[a][l], &dp);
      if (st != PA_OK) return st;
      if (!aligned(dp, 16)) return PA_ERR_INVALID_ARG;
      outp[a][l] = dp;
    }
  }
  void* map_dp = nullptr;
  pa_status st = pa::device_view(block_mapping, &map_dp);
  if (st != PA_OK) return st;
  void* err_dp = nullptr;
  if (dev_error) {
    st = pa::device_view(dev_error, &err_dp);
    if (st != PA_OK) return st;
  }
  const int64_t block_bytes = (int64_t)num_kv_heads * PA_BLOCK_SIZE * head_dim * 2;
  cudaError_t e = pa::launch_block_copy(sk, sv, dk, dv, num_layers,
                                        static_cast<const int64_t*>(map_dp), num_pairs,
                                        block_bytes, src_num_blocks, dst_num_blocks,
                                        static_cast<int32_t*>(err_dp),
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

pa_status pa_read_probe(const void* buf, size_t bytes, int32_t method, uint64_t* sink,
                        int32_t* dev_error, void* stream) {
  if (method < 0 || method > 2) return PA_ERR_INVALID_ARG;
  if (bytes == 0) return PA_OK;
  if (!buf || !sink || !aligned(buf, 16) || bytes % 16 || !aligned(sink, 8) ||
      (dev_error && !aligned(dev_error, 4)))
    return PA_ERR_INVALID_ARG;
  if (method == 2) {
    // whole 4 KiB tiles, an even number of them (two per stage)
    const int64_t n_tiles = (int64_t)(bytes / 4096) & ~(int64_t)1;
    if (n_tiles < 2 || n_tiles > (int64_t(1) << 31)) return PA_ERR_INVALID_ARG;
    CUtensorMap tm;
    pa_status st = encode_pool_map(&tm, buf, n_tiles, 1, 128, PA_DTYPE_BF16);
    if (st != PA_OK) return st;
    // a stride near n / golden ratio, coprime with n: consecutive reads land
    // far apart, and every tile is read once
    int64_t stride = (int64_t)((double)n_tiles * 0.6180339887) | 1;
    auto gcd = [](int64_t a, int64_t b) { while (b) { const int64_t t = a % b; a = b; b = t; } return a; };
    while (gcd(stride, n_tiles) != 1) stride += 2;
    cudaError_t e = pa::launch_read_probe_scattered(
        tm, n_tiles, stride % n_tiles, n_tiles / 3, reinterpret_cast<unsigned long long*>(sink),
        dev_error, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_fail(e);
  }
  cudaError_t e = pa::launch_read_probe(buf, bytes, method,
                                        reinterpret_cast<unsigned long long*>(sink), dev_error,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

}  // extern "C"
