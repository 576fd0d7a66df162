// pa_decode_static.cu -- pa_decode for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc: a plugin running
// inside a host application that owns every byte of device memory and forbids
// its plugins from allocating, or a latency-critical caller for which
// cudaMalloc / cudaFree (which can synchronise the whole device) are not
// acceptable in the decode loop. pa_decode needs scratch memory for its
// split-K partial results, and normally the caller provides it. This entry
// point instead uses a fixed scratch array compiled into the library: it is
// created in each GPU's memory when the library's device code is loaded on
// that GPU and is held until the process exits.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress -- in host code the
// array's name only stands for it and must never be handed to a kernel. Make
// that first call before any stream capture on that device.
//
// Sharing: every call on a device uses the same array. Each call writes every
// partial result it later reads, so nothing has to start at zero, but two
// calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on the array. Order them on one stream, or by events.
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

static __device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up once
// per device.
pa_status scratch_on_current_device(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return pa::record_cuda_error(e);
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_static(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      int32_t block_table_stride, const int32_t* context_lens,
                                      int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                                      int32_t head_dim, int32_t block_size, int64_t num_blocks,
                                      int32_t max_context_len, float scale,
                                      int32_t partition_tokens, int32_t* dev_error,
                                      pa_dtype dtype, void* stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                               partition_tokens);
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  pa_status st = scratch_on_current_device(&scratch);
  if (st != PA_OK) return st;
  return pa_decode(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                   num_seqs, num_q_heads, group_size, head_dim, block_size, num_blocks,
                   max_context_len, scale, partition_tokens, scratch, PA_STATIC_WORKSPACE_BYTES,
                   dev_error, dtype, stream);
}
