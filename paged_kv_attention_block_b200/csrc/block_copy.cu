// copy_block_prefix: copy the first n tokens of pool blocks into other blocks
// (deep dive §11, partial reuse with copy_on_partial_reuse: the matched tokens
// of a partially matching block are copied into a new block).
//
// A pool block holds, per layer, K then V, per KV head, block_size token rows
// of head_dim values, so slots 0 .. n-1 of one (block, layer, K|V, head) are
// one contiguous run of n * head_dim elements.  One warp per (copy, layer,
// K|V, head) run moves it in 16-byte pieces (row bytes are multiples of 16 for
// head_dim 64 / 128 and every pool dtype).  An NVFP4 run holds block_size rows of
// codes and then block_size rows of block scales: the first n of each are copied
// (the scale rows in 8-byte pieces).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace pkv {

struct CopyArgs {
  uint8_t* pool;
  int64_t num_blocks;
  int32_t runs_per_block;  // num_layers * 2 * Hkv
  int32_t log2_block;
  int32_t row_bytes;       // head_dim * element size (NVFP4: head_dim / 2 bytes of codes)
  int32_t scale_row_bytes; // NVFP4: head_dim / 16 bytes of block scales per row, else 0
  const int32_t* src;
  const int32_t* dst;
  const int32_t* n_tokens;
  int32_t count;
  int32_t* status;
};

__global__ void __launch_bounds__(256) copy_block_prefix_kernel(CopyArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t runs = int64_t(a.count) * a.runs_per_block;
  for (int64_t u = int64_t(blockIdx.x) * 8 + warp; u < runs; u += int64_t(gridDim.x) * 8) {
    const int i = int(u / a.runs_per_block), run = int(u % a.runs_per_block);
    const int src = __ldg(a.src + i), dst = __ldg(a.dst + i), n = __ldg(a.n_tokens + i);
    if (src < 0 || src >= a.num_blocks || dst < 0 || dst >= a.num_blocks) {
      if (lane == 0 && run == 0) report(a.status, PKV_DEV_BAD_BLOCK_ID);
      continue;
    }
    if (n < 0 || n > (1 << a.log2_block)) {
      if (lane == 0 && run == 0) report(a.status, PKV_DEV_BAD_COPY);
      continue;
    }
    if (src == dst || n == 0) continue;
    const int64_t codes_bytes = int64_t(a.row_bytes) << a.log2_block;
    const int64_t run_bytes = codes_bytes + (int64_t(a.scale_row_bytes) << a.log2_block);  // one (layer, K|V, head)
    const int64_t block_bytes = run_bytes * a.runs_per_block;
    const uint8_t* sbase = a.pool + src * block_bytes + run * run_bytes;
    uint8_t* dbase = a.pool + dst * block_bytes + run * run_bytes;
    const uint4* s = reinterpret_cast<const uint4*>(sbase);
    uint4* d = reinterpret_cast<uint4*>(dbase);
    const int chunks = n * a.row_bytes / 16;
    for (int c = lane; c < chunks; c += 32) d[c] = __ldg(s + c);
    if (a.scale_row_bytes) {
      const uint2* ss = reinterpret_cast<const uint2*>(sbase + codes_bytes);
      uint2* ds = reinterpret_cast<uint2*>(dbase + codes_bytes);
      for (int c = lane; c < n * a.scale_row_bytes / 8; c += 32) ds[c] = __ldg(ss + c);
    }
  }
}

}  // namespace pkv

extern "C" pkv_status pkv_copy_block_prefix(const pkv_cache* cache, const int32_t* src_blocks,
                                            const int32_t* dst_blocks, const int32_t* n_tokens, int32_t count,
                                            int32_t* dev_status, void* stream) {
  using namespace pkv;
  if (!cache) return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: cache is NULL");
  const pkv_cache& c = *cache;
  if (count < 0) return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: count < 0");
  if (!pkv_is_pow2(c.block_size) || c.block_size < 2)
    return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: block_size %d is not a power of two > 1", c.block_size);
  if (c.head_dim != 64 && c.head_dim != 128) return pkv_fail(PKV_ERR_UNSUPPORTED, "copy_block_prefix: head_dim %d", c.head_dim);
  if (c.num_kv_heads <= 0 || c.num_layers <= 0 || c.num_blocks <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: bad cache shape");
  if (c.kv_dtype < PKV_F32 || c.kv_dtype > PKV_NVFP4) return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: kv_dtype");
  if (c.kv_dtype == PKV_NVFP4 && c.head_dim != 128)
    return pkv_fail(PKV_ERR_UNSUPPORTED, "copy_block_prefix: NVFP4 pools take head_dim 128");
  if (count == 0) return PKV_OK;
  if (!c.pool || !src_blocks || !dst_blocks || !n_tokens)
    return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: null pointer");
  if (reinterpret_cast<uintptr_t>(c.pool) & 15) return pkv_fail(PKV_ERR_INVALID_ARG, "copy_block_prefix: pool not 16-byte aligned");
  const bool fp4 = c.kv_dtype == PKV_NVFP4;
  const int elem = c.kv_dtype == PKV_F32 ? 4 : (c.kv_dtype == PKV_FP8_E4M3 ? 1 : 2);
  CopyArgs a{static_cast<uint8_t*>(c.pool), c.num_blocks, c.num_layers * 2 * c.num_kv_heads, pkv_log2(c.block_size),
             fp4 ? c.head_dim / 2 : c.head_dim * elem, fp4 ? c.head_dim / 16 : 0, src_blocks, dst_blocks, n_tokens,
             count, dev_status};
  const int64_t runs = int64_t(count) * a.runs_per_block;
  const int grid = int(std::min<int64_t>((runs + 7) / 8, 148 * 16));
  copy_block_prefix_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "copy_block_prefix: launch failed: %s", cudaGetErrorString(e));
  return PKV_OK;
}
