// split_kv_reduce: merge partial softmax states over disjoint key sets.
//
// For one output row with parts (o_i normalised, lse_i natural log):
//   M = max_i lse_i, w_i = exp(lse_i - M), o = sum w_i o_i / sum w_i,
//   lse = M + ln sum w_i; parts with lse = -inf weigh nothing.
// Two launch forms share the per-element merge: the public dense form
// ([n_split][rows][d] partials) and the plan-driven form that finishes a paged
// attention launch whose key ranges were split (ragged part lists per tile).
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_args.h"
#include "common.cuh"
#include "internal.h"

namespace pkv {

__global__ void __launch_bounds__(256) dense_reduce_kernel(const float* __restrict__ po, const float* __restrict__ pl,
                                                           int n, int64_t rows, int d, void* out, int out_dtype,
                                                           float* out_lse) {
  const int64_t total = rows * d;
  for (int64_t x = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; x < total; x += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = x / d;
    float o, lse;
    merge_elem(
        n, [&](int i) { return pl[i * rows + r]; }, [&](int i) { return po[i * total + x]; }, o, lse);
    store_any(out, out_dtype, x, o);
    if (out_lse && x % d == 0) out_lse[r] = lse;
  }
}

// One warp per output row of a merge (a merge covers n_q tokens x g heads; the
// CTA at blockIdx.y takes its rows 16 y .. 16 y + 15, four a warp, so a merge of
// 128-row partials spreads over 8 CTAs); lane j merges head dims [VEC j, VEC (j + 1))
// with the same per-element arithmetic as merge_elem, so each lane issues VEC-wide
// loads of the parts.  Latency, not bandwidth, sets this kernel's time: the merges and
// their part lists (staged before the attention kernels started, which waited for the
// staging) are read before the wait for the attention kernels, and a row of two parts
// loads both at once.  40 registers: 12 CTAs an SM (1,776 on a B200) hold most plans' merges at once.
template <int D>
PKV_DEVICE void load_part(const float* part_o, int64_t prow, int lane, float (&x)[D / 32]) {
  constexpr int VEC = D / 32;
  const float* src = part_o + prow * D + lane * VEC;
  if constexpr (VEC == 4) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(src));
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else {
    const float2 f = __ldg(reinterpret_cast<const float2*>(src));
    x[0] = f.x; x[1] = f.y;
  }
}

template <int D>
__global__ void __launch_bounds__(128, 12) plan_reduce_kernel(const ReduceArgs a) {
  constexpr int VEC = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int e = blockIdx.x;
  PkvReduce red{};
  int32_t my_part = 0;  // lane i: the merge's part i (i < 32)
  auto fetch = [&](int m) {
    red = a.reduces[m];
    my_part = lane < red.n_parts ? __ldg(a.parts + red.parts_begin + lane) : 0;
  };
  if (e < a.n_reduce) fetch(e);
  pdl_wait();  // launched as a dependent of the attention kernels: their partial states are complete
  for (; e < a.n_reduce; e += gridDim.x) {
    if (e != int(blockIdx.x)) fetch(e);
    const int R = red.n_q * a.g;
    const int n = red.n_parts;
    const int r_end = min(R, int(blockIdx.y) * 16 + 16);
    for (int r = int(blockIdx.y) * 16 + warp; r < r_end; r += 4) {
      float o[VEC], lse;
      if (n <= 2) {
        // The usual case (a split in two, or a shared-prefix group part and a member's own part):
        // both parts' sums and rows are loaded at once.
        const int64_t p0 = int64_t(__shfl_sync(0xffffffffu, my_part, 0)) + r;
        const int64_t p1 = int64_t(__shfl_sync(0xffffffffu, my_part, 1)) + r;
        const float l0 = n > 0 ? __ldg(a.part_lse + p0) : -INFINITY;
        const float l1 = n > 1 ? __ldg(a.part_lse + p1) : -INFINITY;
        float x0[VEC], x1[VEC];
        if (n > 0) load_part<D>(a.part_o, p0, lane, x0);
        if (n > 1) load_part<D>(a.part_o, p1, lane, x1);
        const float M = fmaxf(l0, l1);
        if (M == -INFINITY) {
#pragma unroll
          for (int v = 0; v < VEC; ++v) o[v] = 0.f;
          lse = -INFINITY;
        } else {
          float num[VEC], den = 0.f;
#pragma unroll
          for (int v = 0; v < VEC; ++v) num[v] = 0.f;
          if (l0 != -INFINITY) {
            const float w = expf(l0 - M);
            den += w;
#pragma unroll
            for (int v = 0; v < VEC; ++v) num[v] = fmaf(w, x0[v], num[v]);
          }
          if (l1 != -INFINITY) {
            const float w = expf(l1 - M);
            den += w;
#pragma unroll
            for (int v = 0; v < VEC; ++v) num[v] = fmaf(w, x1[v], num[v]);
          }
#pragma unroll
          for (int v = 0; v < VEC; ++v) o[v] = num[v] / den;
          lse = M + logf(den);
        }
      } else {
        const int32_t* parts = a.parts + red.parts_begin;
        float M = -INFINITY;
        for (int i = 0; i < n; ++i) M = fmaxf(M, __ldg(a.part_lse + int64_t(__ldg(parts + i)) + r));
        float num[VEC], den = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) num[v] = 0.f;
        for (int i = 0; i < n; ++i) {
          const int64_t prow = int64_t(__ldg(parts + i)) + r;
          const float li = __ldg(a.part_lse + prow);
          if (li == -INFINITY) continue;
          const float w = expf(li - M);
          den += w;
          float x[VEC];
          load_part<D>(a.part_o, prow, lane, x);
#pragma unroll
          for (int v = 0; v < VEC; ++v) num[v] = fmaf(w, x[v], num[v]);
        }
        // M = -inf leaves den = 0: o = 0, lse = -inf, as merge_elem gives.
#pragma unroll
        for (int v = 0; v < VEC; ++v) o[v] = M == -INFINITY ? 0.f : num[v] / den;
        lse = M == -INFINITY ? -INFINITY : M + logf(den);
      }
      const int64_t orow = (int64_t(red.q_begin) + r / a.g) * a.hq + red.kv_head * a.g + r % a.g;
#pragma unroll
      for (int v = 0; v < VEC; ++v) store_any(a.out, a.out_dtype, orow * D + lane * VEC + v, o[v]);
      if (a.out_lse && lane == 0) a.out_lse[orow] = lse;
    }
  }
}

// Plan staging: each thread copies one 16-byte piece of the page-locked host plan (read through
// its device alias) into the workspace.  The grid may start while the kernel ahead of it runs
// (programmatic serialization) and waits for that kernel before it finishes, so the attention
// kernels, which wait for this grid, also see everything written before it on the stream.
__global__ void __launch_bounds__(256) plan_stage_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         int n16) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n16) dst[i] = src[i];
  pdl_wait();
}

cudaError_t launch_plan_stage(const void* plan_dev, void* dst, uint64_t bytes, cudaStream_t st) {
  const int n16 = int(bytes / 16);
  const cudaError_t e = launch_pdl(plan_stage_kernel, dim3((n16 + 255) / 256), dim3(256), 0, st,
                                   static_cast<const uint4*>(plan_dev), static_cast<uint4*>(dst), n16);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_plan_reduce(const ReduceArgs& r, int max_rows, cudaStream_t st) {
  if (r.n_reduce <= 0) return cudaSuccess;
  const dim3 grid(std::min(r.n_reduce, 148 * 16), std::max(1, (max_rows + 15) / 16));
  const cudaError_t e = r.head_dim == 128 ? launch_pdl(plan_reduce_kernel<128>, grid, dim3(128), 0, st, r)
                                           : launch_pdl(plan_reduce_kernel<64>, grid, dim3(128), 0, st, r);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv

extern "C" pkv_status pkv_split_kv_reduce(const float* partial_o, const float* partial_lse, int32_t n_split,
                                          int64_t rows, int32_t head_dim, void* out, int32_t out_dtype,
                                          float* out_lse, void* stream) {
  if (n_split < 0 || rows < 0 || head_dim <= 0) return pkv_fail(PKV_ERR_INVALID_ARG, "split_kv_reduce: negative sizes");
  if (out_dtype != PKV_F32 && out_dtype != PKV_BF16 && out_dtype != PKV_F16)
    return pkv_fail(PKV_ERR_INVALID_ARG, "split_kv_reduce: out_dtype must be F32, BF16 or F16");
  if (rows == 0) return PKV_OK;
  if (!out || (n_split > 0 && (!partial_o || !partial_lse)))
    return pkv_fail(PKV_ERR_INVALID_ARG, "split_kv_reduce: null pointer");
  const int64_t total = rows * head_dim;
  const int grid = int(std::min<int64_t>((total + 255) / 256, 148 * 16));
  pkv::dense_reduce_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(partial_o, partial_lse, n_split, rows,
                                                                                 head_dim, out, out_dtype, out_lse);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "split_kv_reduce: launch failed: %s", cudaGetErrorString(e));
  return PKV_OK;
}
