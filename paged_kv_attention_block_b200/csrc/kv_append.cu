// kv_append: scatter new tokens' K/V rows into their pool slots through the
// block tables (deep dive §2: decode writes the new token's KV; §8: a prefill
// chunk appends its KV before the next chunk; concept explainer "技术原理":
// page-table lookup on KV writes).  fp8 pools store E4M3(x / scale) with
// round-to-nearest-even and saturation (deep dive §13, fp8 KV cache).
//
// One thread moves one 8-element chunk of one (token, K|V, head) row: the
// bytes are tiny next to attention, so the kernel only needs coalesced 8..32 B
// accesses and a grid sized from the element count.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace pkv {

struct AppendArgs {
  void* pool;
  int64_t num_blocks;
  int32_t num_layers, layer, hkv, head_dim, log2_block;
  const void* k_new;
  const void* v_new;
  const int32_t* cu_new;
  const int32_t* start_pos;
  const int32_t* block_tables;
  int32_t max_blocks, num_seqs, total_new;
  const float* k_scale;
  const float* v_scale;
  int32_t* status;
};

template <typename T>
PKV_DEVICE void load8(const T* src, float* x);
template <>
PKV_DEVICE void load8<float>(const float* src, float* x) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 b = reinterpret_cast<const float4*>(src)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
PKV_DEVICE void load8<__nv_bfloat16>(const __nv_bfloat16* src, float* x) {
  const uint4 a = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16_bits_to_float(uint16_t(w[i] & 0xffff));
    x[2 * i + 1] = bf16_bits_to_float(uint16_t(w[i] >> 16));
  }
}
template <>
PKV_DEVICE void load8<__half>(const __half* src, float* x) {
  const uint4 a = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = f16_bits_to_float(uint16_t(w[i] & 0xffff));
    x[2 * i + 1] = f16_bits_to_float(uint16_t(w[i] >> 16));
  }
}

// Find s with cu[s] <= t < cu[s+1] (cu nondecreasing, cu[0] = 0).
PKV_DEVICE int find_seq(const int32_t* cu, int n, int t) {
  int lo = 0, hi = n;  // invariant: cu[lo] <= t < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// Same dtype in and out: move 16 bytes per thread.  ElemT is the element
// type; the chunk holds 16 / sizeof(ElemT) elements.
template <int ELEM>
__global__ void __launch_bounds__(256) kv_append_copy_kernel(AppendArgs a) {
  constexpr int PER = 16 / ELEM;
  const int chunks = a.head_dim / PER;
  const int64_t total = int64_t(a.total_new) * 2 * a.hkv * chunks;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total; idx += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = idx;
    const int c = int(r % chunks); r /= chunks;
    const int h = int(r % a.hkv); r /= a.hkv;
    const int which = int(r % 2);
    const int t = int(r / 2);
    const int s = find_seq(a.cu_new, a.num_seqs, t);
    const int p = __ldg(a.start_pos + s) + (t - __ldg(a.cu_new + s));
    if (p < 0) { report(a.status, PKV_DEV_BAD_APPEND); continue; }
    const int lb = p >> a.log2_block;
    if (lb >= a.max_blocks) { report(a.status, PKV_DEV_BAD_LOGICAL_BLOCK); continue; }
    const int phys = __ldg(a.block_tables + int64_t(s) * a.max_blocks + lb);
    if (phys < 0 || phys >= a.num_blocks) { report(a.status, PKV_DEV_BAD_BLOCK_ID); continue; }
    const int slot = p & ((1 << a.log2_block) - 1);
    const int64_t row = (((int64_t(phys) * a.num_layers + a.layer) * 2 + which) * a.hkv + h) * (int64_t(1) << a.log2_block) + slot;
    const char* src = static_cast<const char*>(which ? a.v_new : a.k_new) + ((int64_t(t) * a.hkv + h) * a.head_dim + c * PER) * ELEM;
    char* dst = static_cast<char*>(a.pool) + (row * a.head_dim + c * PER) * ELEM;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

// fp8 pool: 8 values per thread, quotient x / scale in float32, E4M3 RNE satfinite.
template <typename Tin>
__global__ void __launch_bounds__(256) kv_append_e4m3_kernel(AppendArgs a) {
  const int chunks = a.head_dim / 8;
  const int64_t total = int64_t(a.total_new) * 2 * a.hkv * chunks;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total; idx += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = idx;
    const int c = int(r % chunks); r /= chunks;
    const int h = int(r % a.hkv); r /= a.hkv;
    const int which = int(r % 2);
    const int t = int(r / 2);
    const int s = find_seq(a.cu_new, a.num_seqs, t);
    const int p = __ldg(a.start_pos + s) + (t - __ldg(a.cu_new + s));
    if (p < 0) { report(a.status, PKV_DEV_BAD_APPEND); continue; }
    const int lb = p >> a.log2_block;
    if (lb >= a.max_blocks) { report(a.status, PKV_DEV_BAD_LOGICAL_BLOCK); continue; }
    const int phys = __ldg(a.block_tables + int64_t(s) * a.max_blocks + lb);
    if (phys < 0 || phys >= a.num_blocks) { report(a.status, PKV_DEV_BAD_BLOCK_ID); continue; }
    const int slot = p & ((1 << a.log2_block) - 1);
    const int64_t row = (((int64_t(phys) * a.num_layers + a.layer) * 2 + which) * a.hkv + h) * (int64_t(1) << a.log2_block) + slot;
    const Tin* src = static_cast<const Tin*>(which ? a.v_new : a.k_new) + (int64_t(t) * a.hkv + h) * a.head_dim + c * 8;
    const float scale = __ldg((which ? a.v_scale : a.k_scale) + a.layer * a.hkv + h);
    float x[8];
    load8<Tin>(src, x);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = make_float2(__fdiv_rn(x[2 * i], scale), __fdiv_rn(x[2 * i + 1], scale));
      const uint32_t two = uint32_t(__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3));
      if (i < 2) lo |= two << (16 * i); else hi |= two << (16 * (i - 2));
    }
    uint8_t* dst = static_cast<uint8_t*>(a.pool) + row * a.head_dim + c * 8;
    *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
  }
}

}  // namespace pkv

extern "C" pkv_status pkv_kv_append(const pkv_cache* cache, const void* k_new, const void* v_new, int32_t in_dtype,
                                    const int32_t* cu_new, const int32_t* start_pos, const int32_t* block_tables,
                                    int32_t max_blocks, int32_t num_seqs, int32_t total_new, int32_t* dev_status,
                                    void* stream) {
  using namespace pkv;
  if (!cache) return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: cache is NULL");
  const pkv_cache& c = *cache;
  if (num_seqs < 0 || total_new < 0) return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: negative sizes");
  if (!pkv_is_pow2(c.block_size) || c.block_size < 2)
    return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: block_size %d is not a power of two > 1", c.block_size);
  if (c.head_dim != 64 && c.head_dim != 128) return pkv_fail(PKV_ERR_UNSUPPORTED, "kv_append: head_dim %d", c.head_dim);
  if (c.num_kv_heads <= 0 || c.num_layers <= 0 || c.layer < 0 || c.layer >= c.num_layers || c.num_blocks <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: bad cache shape");
  if (c.kv_dtype < PKV_F32 || c.kv_dtype > PKV_FP8_E4M3) return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: kv_dtype");
  if (c.kv_dtype == PKV_FP8_E4M3) {
    if (in_dtype != PKV_F32 && in_dtype != PKV_BF16 && in_dtype != PKV_F16)
      return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: fp8 pool takes F32, BF16 or F16 values");
    if (!c.k_scale || !c.v_scale) return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: fp8 pool needs k_scale and v_scale");
  } else if (in_dtype != c.kv_dtype) {
    return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: in_dtype %d must equal the pool dtype %d", in_dtype, c.kv_dtype);
  }
  if (total_new == 0 || num_seqs == 0) return PKV_OK;
  if (!c.pool || !k_new || !v_new || !cu_new || !start_pos || !block_tables || max_blocks <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: null pointer or max_blocks <= 0");
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) | reinterpret_cast<uintptr_t>(c.pool)) & 15)
    return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: k_new, v_new and pool must be 16-byte aligned");

  AppendArgs a{c.pool, c.num_blocks, c.num_layers, c.layer, c.num_kv_heads, c.head_dim, pkv_log2(c.block_size),
               k_new, v_new, cu_new, start_pos, block_tables, max_blocks, num_seqs, total_new,
               c.k_scale, c.v_scale, dev_status};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int per = c.kv_dtype == PKV_FP8_E4M3 ? 8 : 16 / (c.kv_dtype == PKV_F32 ? 4 : 2);
  const int64_t work = int64_t(total_new) * 2 * c.num_kv_heads * (c.head_dim / per);
  const int grid = int(std::min<int64_t>((work + 255) / 256, 148 * 16));
  switch (c.kv_dtype) {
    case PKV_F32: kv_append_copy_kernel<4><<<grid, 256, 0, st>>>(a); break;
    case PKV_BF16:
    case PKV_F16: kv_append_copy_kernel<2><<<grid, 256, 0, st>>>(a); break;
    default:
      if (in_dtype == PKV_F32) kv_append_e4m3_kernel<float><<<grid, 256, 0, st>>>(a);
      else if (in_dtype == PKV_BF16) kv_append_e4m3_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
      else kv_append_e4m3_kernel<__half><<<grid, 256, 0, st>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "kv_append: launch failed: %s", cudaGetErrorString(e));
  return PKV_OK;
}
