// pa_read_probe.cu -- the streaming-read ceiling of the GPU's memory.
//
// The decode path only reads the KV cache; the roofline it is held against is
// how fast this GPU can stream bytes from HBM into its SMs and discard them.
// A read+write copy benchmark moves twice the bytes per byte of progress and
// is not that ceiling. Two probes, both reading every byte once:
//   method 0: 128-bit loads that bypass L1, eight in flight per thread, a
//             grid-stride sweep by every resident thread; the words are
//             XOR-folded so the loads cannot be dropped;
//   method 1: bulk asynchronous copies (cp.async.bulk, into this CTA only) of 16 KiB
//             chunks into a 6-stage shared-memory ring per CTA, mbarrier
//             tracked -- the same engine the decode kernels read tiles with.
//   method 2: scattered 4 KiB tiles by 2 KiB TMA tensor boxes, in the decode
//             kernel's CTA shape (the paged-read ceiling; below).
// One atomic XOR per CTA into *sink. All waits are bounded.
#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kVecThreads = 512;
constexpr int kVecUnroll = 8;  // loads in flight per thread (ld_stream8)
constexpr int kBulkChunk = 16384;
constexpr int kBulkStages = 6;
constexpr int kBulkSmem = kBulkChunk * kBulkStages;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Eight 128-bit loads issued back to back (one asm block, so all eight are in
// flight before any result is used), at p, p + s, ..., p + 7s.
__device__ __forceinline__ void ld_stream8(const uint4* p, uint64_t s, uint4 (&v)[8]) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%32];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%4, %5, %6, %7}, [%33];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%8, %9, %10, %11}, [%34];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%12, %13, %14, %15}, [%35];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%16, %17, %18, %19}, [%36];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%20, %21, %22, %23}, [%37];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%24, %25, %26, %27}, [%38];\n\t"
      "ld.global.nc.L1::no_allocate.v4.u32 {%28, %29, %30, %31}, [%39];"
      : "=r"(v[0].x), "=r"(v[0].y), "=r"(v[0].z), "=r"(v[0].w), "=r"(v[1].x), "=r"(v[1].y),
        "=r"(v[1].z), "=r"(v[1].w), "=r"(v[2].x), "=r"(v[2].y), "=r"(v[2].z), "=r"(v[2].w),
        "=r"(v[3].x), "=r"(v[3].y), "=r"(v[3].z), "=r"(v[3].w), "=r"(v[4].x), "=r"(v[4].y),
        "=r"(v[4].z), "=r"(v[4].w), "=r"(v[5].x), "=r"(v[5].y), "=r"(v[5].z), "=r"(v[5].w),
        "=r"(v[6].x), "=r"(v[6].y), "=r"(v[6].z), "=r"(v[6].w), "=r"(v[7].x), "=r"(v[7].y),
        "=r"(v[7].z), "=r"(v[7].w)
      : "l"(p), "l"(p + s), "l"(p + 2 * s), "l"(p + 3 * s), "l"(p + 4 * s), "l"(p + 5 * s),
        "l"(p + 6 * s), "l"(p + 7 * s));
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void fold_into_sink(uint32_t acc, unsigned long long* sink) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t warp_acc[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) warp_acc[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) a ^= warp_acc[w];
    atomicXor(sink, (unsigned long long)a);
  }
}

__global__ void __launch_bounds__(kVecThreads)
    read_vec_kernel(const uint4* __restrict__ p, uint64_t n16, unsigned long long* sink) {
  const uint64_t stride = (uint64_t)gridDim.x * kVecThreads;
  uint64_t i = (uint64_t)blockIdx.x * kVecThreads + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (kVecUnroll - 1) * stride < n16; i += kVecUnroll * stride) {
    uint4 v[kVecUnroll];
    ld_stream8(p + i, stride, v);
#pragma unroll
    for (int k = 0; k < kVecUnroll; ++k) acc ^= v[k].x ^ v[k].y ^ v[k].z ^ v[k].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ld_stream(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  fold_into_sink(acc, sink);
}

// One thread per CTA drives the ring; CTA c takes chunks c, c + grid, ...
__global__ void __launch_bounds__(32)
    read_bulk_kernel(const uint8_t* __restrict__ p, uint64_t bytes, unsigned long long* sink,
                     int32_t* dev_error) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t bars[kBulkStages];
  if (threadIdx.x != 0) return;
  for (int s = 0; s < kBulkStages; ++s) mbar_init(&bars[s], 1);
  fence_barrier_init();
  const uint64_t nchunks = (bytes + kBulkChunk - 1) / kBulkChunk;
  const uint64_t first = blockIdx.x, step = gridDim.x;
  const uint64_t mine = first < nchunks ? (nchunks - 1 - first) / step + 1 : 0;
  auto issue = [&](uint64_t k) {
    const uint64_t off = (first + k * step) * (uint64_t)kBulkChunk;
    const uint32_t sz = (uint32_t)(bytes - off < (uint64_t)kBulkChunk ? bytes - off : kBulkChunk);
    const int st = (int)(k % kBulkStages);
    mbar_arrive_expect_tx(&bars[st], sz);
    bulk_load(ring + st * kBulkChunk, p + off, sz, &bars[st]);
  };
  const uint64_t pro = mine < (uint64_t)kBulkStages ? mine : (uint64_t)kBulkStages;
  for (uint64_t k = 0; k < pro; ++k) issue(k);
  uint32_t acc = 0;
  uint64_t k = 0;
  bool failed = false;
  for (; k < mine; ++k) {
    const int st = (int)(k % kBulkStages);
    if (!mbar_wait(&bars[st], (uint32_t)((k / kBulkStages) & 1))) {
      failed = true;
      break;
    }
    acc ^= *reinterpret_cast<const uint32_t*>(ring + st * kBulkChunk);
    fence_proxy_async_smem();  // the read above precedes the next copy into this stage
    if (k + kBulkStages < mine) issue(k + kBulkStages);
  }
  if (failed) {
    // Let the copies in flight land (each wait bounded) before the CTA exits.
    const uint64_t last = k + kBulkStages < mine ? k + kBulkStages : mine;
    for (uint64_t j = k; j < last; ++j)
      (void)mbar_wait(&bars[j % kBulkStages], (uint32_t)((j / kBulkStages) & 1));
    if (dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
  }
  atomicXor(sink, (unsigned long long)acc);
}

// Method 2: the paged decode's access pattern without its arithmetic. The
// buffer is n 4 KiB tiles (16 rows of 256 bytes, like one KV head of one cache
// block at D = 128); global tile i is read at tile (i * stride + offset) mod n
// (stride coprime with n: every tile once, scattered), as two 2 KiB TMA boxes
// with the 128-byte swizzle, two tiles per stage, in the decode CTA's shape:
// 4 warps, each with a 2-stage ring, 3 CTAs per SM. Every wait is bounded.
constexpr int kScatWarps = 4;
constexpr int kScatStages = 2;
constexpr int kScatStageBytes = 8192;  // two tiles
constexpr int kScatSmem = kScatWarps * kScatStages * kScatStageBytes + 1024;

__global__ void __launch_bounds__(kScatWarps * 32)
    read_scattered_kernel(const __grid_constant__ CUtensorMap tm, int64_t n_tiles,
                          int64_t stride, int64_t offset, unsigned long long* sink,
                          int32_t* dev_error) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t bars[kScatWarps * kScatStages];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = base + warp * kScatStages * kScatStageBytes;
  uint64_t* wb = bars + warp * kScatStages;
  // this warp's pairs of tiles: p = gw, gw + nw, ... (pair p = tiles 2p, 2p+1)
  const int64_t gw = (int64_t)blockIdx.x * kScatWarps + warp;
  const int64_t nw = (int64_t)gridDim.x * kScatWarps;
  const int64_t n_pairs = n_tiles / 2;
  const int64_t mine = gw < n_pairs ? (n_pairs - 1 - gw) / nw + 1 : 0;
  if (lane == 0) {
    for (int st = 0; st < kScatStages; ++st) mbar_init(&wb[st], 1);
    fence_barrier_init();
  }
  __syncwarp();
  auto tile_of = [&](int64_t i) { return (int)((i * stride + offset) % n_tiles); };
  auto issue = [&](int64_t k) {  // lane 0
    const int st = (int)(k % kScatStages);
    uint8_t* dst = ring + st * kScatStageBytes;
    const int64_t p = gw + k * nw;
    mbar_arrive_expect_tx(&wb[st], kScatStageBytes);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int tile = tile_of(2 * p + t);
      tma_load_4d(dst + t * 4096, &tm, &wb[st], 0, 0, 0, tile);
      tma_load_4d(dst + t * 4096 + 2048, &tm, &wb[st], 64, 0, 0, tile);
    }
  };
  if (lane == 0)
    for (int64_t k = 0; k < mine && k < kScatStages; ++k) issue(k);
  uint32_t acc = 0;
  int64_t k = 0;
  bool failed = false;
  for (; k < mine; ++k) {
    const int st = (int)(k % kScatStages);
    if (!__all_sync(0xffffffffu, mbar_wait(&wb[st], (uint32_t)((k / kScatStages) & 1)))) {
      failed = true;
      break;
    }
    acc ^= *reinterpret_cast<const uint32_t*>(ring + st * kScatStageBytes + lane * 256);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && k + kScatStages < mine) issue(k + kScatStages);
  }
  if (failed) {
    // Let the copies in flight land (each wait bounded) before the CTA exits.
    const int64_t last = k + kScatStages < mine ? k + kScatStages : mine;
    for (int64_t j = k; j < last; ++j)
      (void)mbar_wait(&wb[j % kScatStages], (uint32_t)((j / kScatStages) & 1));
    if (lane == 0 && dev_error) atomicAdd(dev_error, PA_DEV_ERR_TIMEOUT);
  }
  fold_into_sink(acc, sink);
}

}  // namespace

cudaError_t launch_read_probe_scattered(const CUtensorMap& tm, int64_t n_tiles, int64_t stride,
                                        int64_t offset, unsigned long long* sink,
                                        int32_t* dev_error, cudaStream_t stream) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  e = cudaFuncSetAttribute(read_scattered_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kScatSmem);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, read_scattered_kernel,
                                                    kScatWarps * 32, kScatSmem);
  if (e != cudaSuccess) return e;
  const int grid = sms * (per_sm > 0 ? per_sm : 1);
  read_scattered_kernel<<<grid, kScatWarps * 32, kScatSmem, stream>>>(tm, n_tiles, stride, offset,
                                                                      sink, dev_error);
  return cudaGetLastError();
}

cudaError_t launch_read_probe(const void* buf, size_t bytes, int method,
                              unsigned long long* sink, int32_t* dev_error,
                              cudaStream_t stream) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if (method == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, read_vec_kernel, kVecThreads, 0);
    if (e != cudaSuccess) return e;
    const int grid = sms * (per_sm > 0 ? per_sm : 1);
    read_vec_kernel<<<grid, kVecThreads, 0, stream>>>(static_cast<const uint4*>(buf), bytes / 16,
                                                      sink);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(read_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kBulkSmem);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, read_bulk_kernel, 32, kBulkSmem);
  if (e != cudaSuccess) return e;
  const int grid = sms * (per_sm > 0 ? per_sm : 1);
  read_bulk_kernel<<<grid, 32, kBulkSmem, stream>>>(static_cast<const uint8_t*>(buf), bytes, sink,
                                                    dev_error);
  return cudaGetLastError();
}

}  // namespace pa
