// kv_append: scatter new tokens' K/V rows into their pool slots through the
// block tables (deep dive §2: decode writes the new token's KV; §8: a prefill
// chunk appends its KV before the next chunk; concept explainer "技术原理":
// page-table lookup on KV writes).  fp8 pools store E4M3(x / scale) with
// round-to-nearest-even and saturation (deep dive §13, fp8 KV cache); NVFP4
// pools (deep dive §13, NVFP4 KV cache) store per 16-value group an E4M3 block
// scale of max|x| / (6 g) and E2M1 codes of x / (scale g), g the float32 scale
// of the (layer, KV head, K|V).
//
// One warp per (token, K|V): lane 0 resolves the destination slot once (the
// token's sequence by binary search over cu_new staged in shared memory, its
// position, the block table entry), then the lanes move the token's rows for
// every KV head in 16-byte (8-byte for fp8) pieces.  The bytes are tiny next
// to attention; what costs is the chain of dependent index loads, kept to
// three per unit.
#include <cuda_runtime.h>

#include <algorithm>

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

// Packed token t belongs to sequence s with cu[s] <= t < cu[s + 1] (binary search;
// cu is in shared memory when the batch is small enough, else global memory).
PKV_DEVICE int find_seq(const int32_t* cu, int n, int t) {
  int lo = 0, hi = n;  // invariant: cu[lo] <= t < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

constexpr int kCuCache = 2048;  // sequences whose cu_new entries are staged in shared memory

// One warp per (new token, K|V): lane 0 resolves the destination slot (sequence,
// position, block table entry) once, then the warp moves the token's rows for
// every KV head.  Returns the pool element offset of head 0's row, or -1 after
// recording a device error.
PKV_DEVICE int64_t append_target(const AppendArgs& a, const int32_t* cu, int t, int which, int lane) {
  int64_t base = -1;
  if (lane == 0) {
    const int s = find_seq(cu, a.num_seqs, t);
    const int p = __ldg(a.start_pos + s) + (t - cu[s]);
    const int lb = p >> a.log2_block;
    if (p < 0) {
      report(a.status, PKV_DEV_BAD_APPEND);
    } else if (lb >= a.max_blocks) {
      report(a.status, PKV_DEV_BAD_LOGICAL_BLOCK);
    } else {
      const int phys = __ldg(a.block_tables + int64_t(s) * a.max_blocks + lb);
      if (phys < 0 || phys >= a.num_blocks) {
        report(a.status, PKV_DEV_BAD_BLOCK_ID);
      } else {
        const int slot = p & ((1 << a.log2_block) - 1);
        base = ((((int64_t(phys) * a.num_layers + a.layer) * 2 + which) * a.hkv) << a.log2_block) + slot;
        base *= a.head_dim;
      }
    }
  }
  return __shfl_sync(0xffffffffu, base, 0);
}

PKV_DEVICE const int32_t* stage_cu(const AppendArgs& a, int32_t* s_cu) {
  const bool cached = a.num_seqs < kCuCache;
  if (cached)
    for (int i = threadIdx.x; i <= a.num_seqs; i += blockDim.x) s_cu[i] = __ldg(a.cu_new + i);
  __syncthreads();
  return cached ? s_cu : a.cu_new;
}

template <int ELEM>
__global__ void __launch_bounds__(256) kv_append_copy_kernel(AppendArgs a) {
  pdl_trigger();  // a programmatic dependent (the plan staging) may start now; it waits for this grid
  __shared__ int32_t s_cu[kCuCache + 1];
  const int32_t* cu = stage_cu(a, s_cu);
  constexpr int PER = 16 / ELEM;  // elements per 16-byte chunk
  const int row_chunks = a.head_dim / PER;
  const int chunks = a.hkv * row_chunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int u = blockIdx.x * 8 + warp; u < 2 * a.total_new; u += gridDim.x * 8) {
    const int t = u >> 1, which = u & 1;
    const int64_t base = append_target(a, cu, t, which, lane);
    if (base < 0) continue;
    const char* src = static_cast<const char*>(which ? a.v_new : a.k_new) + int64_t(t) * a.hkv * a.head_dim * ELEM;
    char* dst = static_cast<char*>(a.pool) + base * ELEM;
    for (int x = lane; x < chunks; x += 32) {
      const int h = x / row_chunks, c = x % row_chunks;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (int64_t(h) * a.head_dim + c * PER) * ELEM));
      *reinterpret_cast<uint4*>(dst + ((int64_t(h) << a.log2_block) * a.head_dim + c * PER) * ELEM) = v;
    }
  }
}

template <typename Tin>
__global__ void __launch_bounds__(256) kv_append_e4m3_kernel(AppendArgs a) {
  pdl_trigger();  // a programmatic dependent (the plan staging) may start now; it waits for this grid
  __shared__ int32_t s_cu[kCuCache + 1];
  const int32_t* cu = stage_cu(a, s_cu);
  const int row_chunks = a.head_dim / 8;  // 8 values -> 8 bytes
  const int chunks = a.hkv * row_chunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int u = blockIdx.x * 8 + warp; u < 2 * a.total_new; u += gridDim.x * 8) {
    const int t = u >> 1, which = u & 1;
    const int64_t base = append_target(a, cu, t, which, lane);
    if (base < 0) continue;
    const Tin* src = static_cast<const Tin*>(which ? a.v_new : a.k_new) + int64_t(t) * a.hkv * a.head_dim;
    uint8_t* dst = static_cast<uint8_t*>(a.pool) + base;
    const float* scales = (which ? a.v_scale : a.k_scale) + a.layer * a.hkv;
    for (int x = lane; x < chunks; x += 32) {
      const int h = x / row_chunks, c = x % row_chunks;
      const float scale = __ldg(scales + h);
      float v[8];
      load8<Tin>(src + int64_t(h) * a.head_dim + c * 8, v);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 q = make_float2(__fdiv_rn(v[2 * i], scale), __fdiv_rn(v[2 * i + 1], scale));
        const uint32_t two = uint32_t(__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3));
        if (i < 2) lo |= two << (16 * i); else hi |= two << (16 * (i - 2));
      }
      *reinterpret_cast<uint2*>(dst + (int64_t(h) << a.log2_block) * a.head_dim + c * 8) = make_uint2(lo, hi);
    }
  }
}

// float -> E2M1 code: nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6, ties to the even code (the
// thresholds alternate strict and non-strict accordingly), saturating at 6; the sign bit is
// the input's.
PKV_DEVICE uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  const uint32_t c = uint32_t(a > 0.25f) + uint32_t(a >= 0.75f) + uint32_t(a > 1.25f) + uint32_t(a >= 1.75f) +
                     uint32_t(a > 2.5f) + uint32_t(a >= 3.5f) + uint32_t(a > 5.0f);
  return c | ((__float_as_uint(y) >> 31) << 3);
}

template <typename Tin>
PKV_DEVICE void load4(const Tin* src, float* x);
template <>
PKV_DEVICE void load4<float>(const float* src, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
PKV_DEVICE void load4<__nv_bfloat16>(const __nv_bfloat16* src, float* x) {
  const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
  x[0] = bf16_bits_to_float(uint16_t(a.x & 0xffff)); x[1] = bf16_bits_to_float(uint16_t(a.x >> 16));
  x[2] = bf16_bits_to_float(uint16_t(a.y & 0xffff)); x[3] = bf16_bits_to_float(uint16_t(a.y >> 16));
}
template <>
PKV_DEVICE void load4<__half>(const __half* src, float* x) {
  const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
  x[0] = f16_bits_to_float(uint16_t(a.x & 0xffff)); x[1] = f16_bits_to_float(uint16_t(a.x >> 16));
  x[2] = f16_bits_to_float(uint16_t(a.y & 0xffff)); x[3] = f16_bits_to_float(uint16_t(a.y >> 16));
}

// NVFP4 (head_dim 128): one warp per (token, K|V); per KV head each lane quantises four
// consecutive dims, the four lanes of a 16-value group share its max through shuffles, and
// lane 4j writes the group's block scale.
template <typename Tin>
__global__ void __launch_bounds__(256) kv_append_nvfp4_kernel(AppendArgs a) {
  pdl_trigger();  // a programmatic dependent (the plan staging) may start now; it waits for this grid
  __shared__ int32_t s_cu[kCuCache + 1];
  const int32_t* cu = stage_cu(a, s_cu);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t run_bytes = int64_t(128 / 2 + 128 / 16) << a.log2_block;
  for (int u = blockIdx.x * 8 + warp; u < 2 * a.total_new; u += gridDim.x * 8) {
    const int t = u >> 1, which = u & 1;
    const int64_t base = append_target(a, cu, t, which, lane);  // element offset of head 0's row
    if (base < 0) continue;
    const int64_t row = base >> 7;  // (run of head 0) * B + slot
    const int64_t run0 = row >> a.log2_block;
    const int slot = int(row & ((1 << a.log2_block) - 1));
    const Tin* src = static_cast<const Tin*>(which ? a.v_new : a.k_new) + int64_t(t) * a.hkv * 128;
    const float* gs = (which ? a.v_scale : a.k_scale) + a.layer * a.hkv;
    for (int h = 0; h < a.hkv; ++h) {
      float x[4];
      load4<Tin>(src + h * 128 + lane * 4, x);
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const float g = __ldg(gs + h);
      const __nv_fp8_storage_t sc = __nv_cvt_float_to_fp8(__fdiv_rn(amax, __fmul_rn(6.0f, g)), __NV_SATFINITE, __NV_E4M3);
      const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
      uint32_t codes = 0;
      if (s != 0.f) {
        const float den = __fmul_rn(s, g);
#pragma unroll
        for (int i = 0; i < 4; ++i) codes |= e2m1_code(__fdiv_rn(x[i], den)) << (4 * i);
      }
      uint8_t* run = static_cast<uint8_t*>(a.pool) + (run0 + h) * run_bytes;
      *reinterpret_cast<uint16_t*>(run + slot * 64 + lane * 2) = uint16_t(codes);
      if ((lane & 3) == 0) run[(int64_t(64) << a.log2_block) + slot * 8 + (lane >> 2)] = sc;
    }
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
  if (c.kv_dtype < PKV_F32 || c.kv_dtype > PKV_NVFP4) return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: kv_dtype");
  if (c.kv_dtype == PKV_NVFP4 && c.head_dim != 128)
    return pkv_fail(PKV_ERR_UNSUPPORTED, "kv_append: NVFP4 pools take head_dim 128");
  if (c.kv_dtype == PKV_FP8_E4M3 || c.kv_dtype == PKV_NVFP4) {
    if (in_dtype != PKV_F32 && in_dtype != PKV_BF16 && in_dtype != PKV_F16)
      return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: fp8 and NVFP4 pools take F32, BF16 or F16 values");
    if (!c.k_scale || !c.v_scale)
      return pkv_fail(PKV_ERR_INVALID_ARG, "kv_append: fp8 and NVFP4 pools need k_scale and v_scale");
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
  // Eight (token, K|V) units per 256-thread block, one per warp.
  const int grid = int(std::min<int64_t>((int64_t(total_new) * 2 + 7) / 8, 148 * 16));
  switch (c.kv_dtype) {
    case PKV_F32: kv_append_copy_kernel<4><<<grid, 256, 0, st>>>(a); break;
    case PKV_BF16:
    case PKV_F16: kv_append_copy_kernel<2><<<grid, 256, 0, st>>>(a); break;
    case PKV_NVFP4:
      if (in_dtype == PKV_F32) kv_append_nvfp4_kernel<float><<<grid, 256, 0, st>>>(a);
      else if (in_dtype == PKV_BF16) kv_append_nvfp4_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
      else kv_append_nvfp4_kernel<__half><<<grid, 256, 0, st>>>(a);
      break;
    default:
      if (in_dtype == PKV_F32) kv_append_e4m3_kernel<float><<<grid, 256, 0, st>>>(a);
      else if (in_dtype == PKV_BF16) kv_append_e4m3_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
      else kv_append_e4m3_kernel<__half><<<grid, 256, 0, st>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "kv_append: launch failed: %s", cudaGetErrorString(e));
  return PKV_OK;
}
