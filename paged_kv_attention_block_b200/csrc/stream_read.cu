// A plain read-only HBM stream: the practical ceiling the attention kernels'
// bandwidth is compared with.
//
// Decode attention is a read stream (the pages' deep dive, §2: decode reads all
// history KV every step), so its bandwidth is best judged against the fastest
// pure read of the same memory, not only against a copy.  Two forms:
//   * loads: a persistent grid (a multiple of the SM count) of 512-thread CTAs,
//     each thread issuing four independent 16-byte non-caching loads per step
//     over a grid-strided range, folding them into an XOR;
//   * bulk: the form the attention kernels use, one elected thread per CTA
//     issuing 1-dimensional cp.async.bulk copies of 32 KB chunks into a ring of
//     four shared-memory stages whose completion is counted on mbarriers (no
//     multicast); one warp reads a word of each landed chunk.
// Each CTA XOR-folds what it read into *sink, so no load is dead code.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace pkv {

__global__ void __launch_bounds__(512) stream_read_ldg_kernel(const uint4* __restrict__ src, int64_t n16,
                                                              uint32_t* sink) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                   : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                   : "l"(src + i + u * stride));
#pragma unroll
    for (int u = 0; u < 4; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldg(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

constexpr int kBulkChunk = 32 * 1024;
constexpr int kBulkStages = 4;

// Chunks c = blockIdx.x, blockIdx.x + gridDim.x, ... of kBulkChunk bytes (the last one shorter).
__global__ void __launch_bounds__(64) stream_read_bulk_kernel(const uint8_t* __restrict__ src, int64_t bytes,
                                                              uint32_t* sink, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023) & ~1023u;
  const uint32_t bars = base + kBulkStages * kBulkChunk;
  __shared__ volatile int s_abort;
  __shared__ volatile long long s_issued;  // chunks whose copy was issued
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(bars + 8 * s, 1);                  // full: the producer's arrive + the bytes
      mbar_init(bars + 8 * (kBulkStages + s), 1);  // empty: the reader's arrive
    }
    s_abort = 0;
    s_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t nchunks = (bytes + kBulkChunk - 1) / kBulkChunk;
  int64_t mine = 0;
  if (blockIdx.x < nchunks) mine = (nchunks - 1 - blockIdx.x) / gridDim.x + 1;
  if (tid < 32) {
    // producer: lane 0 issues the copies
    if (lane == 0) {
      for (int64_t k = 0; k < mine; ++k) {
        const int s = int(k % kBulkStages);
        if (!mbar_wait(bars + 8 * (kBulkStages + s), uint32_t(((k / kBulkStages) & 1) ^ 1))) {
          report(status, PKV_DEV_TIMEOUT);
          s_abort = 1;
          break;
        }
        const int64_t off = (int64_t(blockIdx.x) + k * gridDim.x) * kBulkChunk;
        const uint32_t n = uint32_t(std::min<int64_t>(kBulkChunk, bytes - off));
        mbar_arrive_expect_tx(bars + 8 * s, n);
        bulk_load_1d(base + s * kBulkChunk, src + off, n, bars + 8 * s);
        s_issued = k + 1;
      }
    }
  } else {
    // reader warp: one word per landed chunk, then release the stage
    uint32_t acc = 0;
    for (int64_t k = 0; k < mine; ++k) {
      const int s = int(k % kBulkStages);
      if (s_abort || !mbar_wait(bars + 8 * s, uint32_t((k / kBulkStages) & 1))) {
        report(status, PKV_DEV_TIMEOUT);
        s_abort = 1;
        break;
      }
      uint32_t w;
      asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(w) : "r"(base + s * kBulkChunk + lane * 4));
      acc ^= w;
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (kBulkStages + s), 1);
    }
    acc = __reduce_xor_sync(0xffffffffu, acc);
    if (lane == 0) atomicXor(sink, acc);
  }
  // Loads still in flight (after an abort) must land before the CTA's shared memory goes away.
  __syncthreads();
  if (tid == 0 && s_abort) {
    const int64_t issued = s_issued;
    for (int64_t k = std::max<int64_t>(0, issued - kBulkStages); k < issued; ++k)
      mbar_wait(bars + 8 * int(k % kBulkStages), uint32_t((k / kBulkStages) & 1));
  }
}

}  // namespace pkv

extern "C" pkv_status pkv_stream_read(const void* src, size_t bytes, int32_t mode, uint32_t* sink,
                                      int32_t* dev_status, void* stream) {
  if (bytes == 0) return PKV_OK;
  if (!src || !sink) return pkv_fail(PKV_ERR_INVALID_ARG, "stream_read: null pointer");
  if ((reinterpret_cast<uintptr_t>(src) | bytes) & 15)
    return pkv_fail(PKV_ERR_INVALID_ARG, "stream_read: src and bytes must be multiples of 16");
  if (mode != 0 && mode != 1) return pkv_fail(PKV_ERR_INVALID_ARG, "stream_read: mode %d (0 loads, 1 bulk)", mode);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "stream_read: device query: %s", cudaGetErrorString(e));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode == 0) {
    pkv::stream_read_ldg_kernel<<<sms * 4, 512, 0, st>>>(static_cast<const uint4*>(src), int64_t(bytes / 16), sink);
  } else {
    const int smem = 1024 + pkv::kBulkStages * pkv::kBulkChunk + 16 * pkv::kBulkStages;
    e = cudaFuncSetAttribute(pkv::stream_read_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "stream_read: %s", cudaGetErrorString(e));
    pkv::stream_read_bulk_kernel<<<sms * 1, 64, smem, st>>>(static_cast<const uint8_t*>(src), int64_t(bytes), sink,
                                                          dev_status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "stream_read: launch failed: %s", cudaGetErrorString(e));
  return PKV_OK;
}
