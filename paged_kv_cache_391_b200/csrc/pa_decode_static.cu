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
// that first call before any stream capture on that device. The address is
// kept per device together with the id of the CUDA context it belongs to;
// when the device's context changes (after cudaDeviceReset, the library's
// device code is loaded again and the array may move) the next call looks
// the address up again.
//
// Sharing: every call on a device uses the same array. Each call writes every
// partial result it later reads, so nothing has to start at zero, but two
// calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on the array. Order them on one stream, or by events.
#include <cudaTypedefs.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

static __device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 128;

struct ScratchSlot {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;  // 0: unknown
};

std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

// Unique id of the calling thread's current CUDA context (driver entry
// points, looked up once); false when there is none or it cannot be read.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

// Device address of g_decode_scratch on the current device, looked up on the
// first call and again whenever the device's context has changed.
pa_status scratch_on_current_device(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (!slot.addr || !have_id || slot.ctx_id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);  // makes the context current if needed
    if (e != cudaSuccess) return pa::record_cuda_error(e);
    unsigned long long now = 0;
    slot.addr = p;
    slot.ctx_id = current_context_id(&now) ? now : 0;
  }
  *addr = slot.addr;
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
