// Paged attention for float32 pools on CUDA cores.
//
// Same work list and output convention as the tensor-core kernel; float32 KV
// asks for float32 accuracy (1e-5), which the 16-bit tensor-core paths cannot
// give, so scores and the softmax run in fp32 FMAs.  One warp handles one row
// (query token x head) at a time; lanes split the head dimension.  This path
// serves small or accuracy-first pools; the bandwidth-bound pools are bf16,
// f16 and fp8 (attn_mma.cu).
#include <cuda_runtime.h>

#include "attn_args.h"
#include "common.cuh"
#include "internal.h"

namespace pkv {

template <int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnArgs a) {
  constexpr int PL = D / 32;  // dims per lane
  __shared__ int s_item;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total_q = __ldg(a.cu_q_lens + a.num_seqs);
  const int bmask = (1 << a.log2_block) - 1;
  const float* pool = static_cast<const float*>(a.pool);
  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(a.counter, 1u));
    __syncthreads();
    const int idx = s_item;
    __syncthreads();
    if (idx >= a.n_items) break;
    const PkvItem it = a.items[idx];
    bool ok = it.seq >= 0 && it.seq < a.num_seqs && it.kv_head >= 0 && it.kv_head < a.hkv && it.n_q > 0 &&
              it.n_q * a.g <= a.max_rows && it.q_begin >= 0 && it.q_begin + it.n_q <= total_q && it.k_begin >= 0 &&
              it.k_begin <= it.k_end;
    if (ok) {
      const int L = __ldg(a.seq_lens + it.seq);
      ok = it.k_end <= L && (it.k_end == 0 || ((it.k_end - 1) >> a.log2_block) < a.max_blocks) &&
           (it.pos0 < 0 || it.pos0 + it.n_q <= L);
    }
    if (!ok) {
      if (tid == 0) report(a.status, PKV_DEV_PLAN_MISMATCH);
      continue;
    }
    const int32_t* bt_row = a.block_tables + int64_t(it.seq) * a.max_blocks;
    const int R = it.n_q * a.g;
    for (int r = warp; r < R; r += 4) {
      const int64_t token = it.q_begin + r / a.g;
      const int head = it.kv_head * a.g + r % a.g;
      const float* qrow = static_cast<const float*>(a.q) + (token * a.hq + head) * D;
      float q[PL], acc[PL];
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        q[i] = qrow[lane + 32 * i];
        acc[i] = 0.f;
      }
      const int lim = it.pos0 >= 0 ? min(it.k_end, it.pos0 + r / a.g + 1) : it.k_end;
      float m = -INFINITY, l = 0.f;
      for (int t = max(it.k_begin, window_start(a.window, it.pos0 >= 0 ? it.pos0 + r / a.g : -1)); t < lim; ++t) {
        const int phys = __ldg(bt_row + (t >> a.log2_block));
        if (phys < 0 || phys >= a.num_blocks) {
          if (lane == 0) report(a.status, PKV_DEV_BAD_BLOCK_ID);
          continue;
        }
        const int64_t rowk =
            ((int64_t(phys) * a.num_layers + a.layer) * 2 * a.hkv + it.kv_head) * (int64_t(1) << a.log2_block) + (t & bmask);
        const float* krow = pool + rowk * D;
        const float* vrow = krow + (int64_t(a.hkv) << a.log2_block) * D;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) dot = fmaf(q[i], krow[lane + 32 * i], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float s = dot * a.softmax_scale;
        const float mnew = fmaxf(m, s);
        const float alpha = expf(m - mnew);
        const float p = expf(s - mnew);
        l = l * alpha + p;
#pragma unroll
        for (int i = 0; i < PL; ++i) acc[i] = fmaf(p, vrow[lane + 32 * i], acc[i] * alpha);
        m = mnew;
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = l > 0.f ? m + logf(l) : -INFINITY;
      if (it.part_row >= 0) {
        const int64_t prow = int64_t(it.part_row) + r;
#pragma unroll
        for (int i = 0; i < PL; ++i) a.part_o[prow * D + lane + 32 * i] = acc[i] * inv;
        if (lane == 0) a.part_lse[prow] = lse;
      } else {
        const int64_t orow = token * a.hq + head;
        float* o = static_cast<float*>(a.out) + orow * D;
#pragma unroll
        for (int i = 0; i < PL; ++i) o[lane + 32 * i] = acc[i] * inv;
        if (lane == 0 && a.out_lse) a.out_lse[orow] = lse;
      }
    }
  }
}

template <int D>
cudaError_t launch_f32(const AttnArgs& a, int grid, cudaStream_t st) {
  attn_f32_kernel<D><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

AttnKernel f32_kernel(int head_dim) {
  if (head_dim == 128) return AttnKernel{reinterpret_cast<const void*>(&attn_f32_kernel<128>), 128, 0, &launch_f32<128>, PKV_TILE_ROWS};
  return AttnKernel{reinterpret_cast<const void*>(&attn_f32_kernel<64>), 128, 0, &launch_f32<64>, PKV_TILE_ROWS};
}

}  // namespace pkv
