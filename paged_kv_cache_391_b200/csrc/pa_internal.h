// pa_internal.h -- launch interfaces between libpa's C ABI (pa_api.cu) and
// its kernel translation units. Not installed; not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

struct DecodeLaunch {
  CUtensorMap tm_k;  // K pool as [NB][H_kv][16][D], 64x16 boxes, 128-byte swizzle
  CUtensorMap tm_v;
  void* out;
  float* part_o;     // [S][H_q][max_parts][D]
  float* part_lse;   // [S][H_q][max_parts]
  const void* q;
  const int32_t* q_start;  // NULL: one query token per sequence (decode)
  int32_t num_q_tokens;    // rows of q / out (= num_seqs for decode)
  int32_t max_query_len;   // 1 for decode
  int32_t max_qtiles;      // 16-row query tiles per (sequence, KV head)
  const int32_t* block_tables;
  int32_t bt_stride;
  const int32_t* context_lens;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t group;
  int32_t head_dim;
  int64_t num_blocks;
  int32_t max_context_len;
  float scale_log2;  // scale * log2(e)
  int32_t part_blocks;
  int32_t part_tokens;
  int32_t max_parts;
  int32_t* dev_error;
  int bf16;          // 0 = fp16, 1 = bf16
  uint32_t* items;   // work queue: [num_seqs * max_parts] (seq << 16) | part
  int32_t* plan;     // [0] = items listed, [1] = work counter
  // tcgen05 chunk path, longest first (NULL: grid order): [max items] of
  // {sequence, pair * max_parts + partition}, then [0] = items listed
  uint2* chunk_items;
  int32_t* chunk_plan;
  // Decode with a shared prefix (pa_decode_shared_prefix): partitions below
  // first_part are computed by the tcgen05 kernel over all sequences at once;
  // the decode kernel starts at first_part. 0 otherwise. shared_tm_q (the
  // query map of that kernel) set: the decode's launch makes it, between the
  // decode kernel and the reduce.
  int32_t first_part;
  const CUtensorMap* shared_tm_q;
};

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream);

// Decode (one query token per sequence) as a plan kernel that lists the
// (sequence, partition) items longest first, a persistent grid that pulls
// them from a counter, and the reduce. Uses a.items and a.plan.
cudaError_t launch_decode_persistent(const DecodeLaunch& a, cudaStream_t stream);

// The log-sum-exp reduce of split partitions alone (no-op for one partition).
cudaError_t launch_reduce(const DecodeLaunch& a, cudaStream_t stream);

// Query chunks on the tcgen05 tensor cores: supported shapes, and the launch
// (partition kernel; the caller runs launch_reduce after it). tm_q maps q as
// [tokens][H_q][D] with boxes of 64 columns x group heads x 128/group tokens.
bool prefill_tc_supported(const DecodeLaunch& a);
// Whether a chunk call takes the tcgen05 path (the same test pa_prefill_chunk
// applies), and the most (sequence, tile pair, partition) items it can have.
bool prefill_tc_eligible(int32_t head_dim, int32_t group, int32_t max_query_len, int64_t parts,
                         int32_t partition_tokens);
int64_t prefill_tc_max_items(int32_t num_seqs, int32_t max_query_len, int32_t group,
                             int64_t parts);
cudaError_t launch_prefill_tc(const DecodeLaunch& a, const CUtensorMap& tm_q, cudaStream_t stream);

// The shared prefix's partitions [0, a.first_part) of every sequence on the
// tcgen05 chunk kernel: the sequences' query tokens (one each, rows of q) as
// the query tokens of one sequence whose context is the first
// a.first_part * a.part_tokens keys of sequence 0's table, without a causal
// mask, each partition's result written as the decode's fp32 partials.
cudaError_t launch_prefill_tc_shared(const DecodeLaunch& a, const CUtensorMap& tm_q,
                                     cudaStream_t stream);
bool prefill_tc_shared_supported(const DecodeLaunch& a);

// Records a CUDA error for pa_last_cuda_error() and returns PA_ERR_CUDA.
pa_status record_cuda_error(cudaError_t e);

// The address a kernel uses for p: device and managed memory as is, pinned or
// registered host memory through its mapped device address. Anything else
// (pageable host memory, an unknown pointer) is PA_ERR_INVALID_ARG.
pa_status device_view(const void* p, void** dev_ptr);

cudaError_t launch_write_kv(const void* k, const void* v, void* k_cache, void* v_cache,
                            const int64_t* slot_mapping, int32_t num_tokens,
                            int32_t num_kv_heads, int32_t head_dim, int64_t num_blocks,
                            int32_t* dev_error, cudaStream_t stream);

cudaError_t launch_block_copy(void* const* src_k, void* const* src_v, void* const* dst_k,
                              void* const* dst_v, int32_t num_layers,
                              const int64_t* block_mapping, int32_t num_pairs,
                              int64_t block_bytes, int64_t src_num_blocks,
                              int64_t dst_num_blocks, int32_t* dev_error, cudaStream_t stream);

// Streaming-read probe (pa_read_probe): method 0 = vector loads, 1 = bulk copies.
cudaError_t launch_read_probe(const void* buf, size_t bytes, int method,
                              unsigned long long* sink, int32_t* dev_error, cudaStream_t stream);
// Method 2: n_tiles 4 KiB tiles of `tm` (a [n][1][16][128] 16-bit pool map)
// read in the order (i * stride + offset) mod n_tiles.
cudaError_t launch_read_probe_scattered(const CUtensorMap& tm, int64_t n_tiles, int64_t stride,
                                        int64_t offset, unsigned long long* sink,
                                        int32_t* dev_error, cudaStream_t stream);

}  // namespace pa
