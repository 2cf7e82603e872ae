// Paged attention on tensor cores for bf16, f16 and fp8-e4m3 KV pools.
//
// What it computes: out = softmax(scale * q K^T) V for every query row, with
// K/V of each sequence read through its block table (deep dive, gentlecold.top,
// §2: decode reads all history KV; §9: blocks of the pool reached through the
// block table), for a packed mix of decode rows and causal prefill chunks in
// one launch (§6, §8).  Query head h reads KV head h / (Hq / Hkv).
//
// How: a persistent grid of 4-warp CTAs pulls work items (rows x key range)
// from an atomic counter.  Each item streams its keys in 64-key tiles through a
// multi-stage shared-memory ring filled with 16-byte cp.async copies (one
// block-table lookup per row, zero fill past the range), and runs the QK^T and
// PV products on m16n8k16 MMAs with fp32 accumulation and an online softmax in
// the exp2 domain.  The Hq/Hkv query heads that share a KV head are rows of
// one tile, so every K/V byte is read once per item.
//   * Items with at most 16 rows (decode): the 4 warps take a quarter of the
//     keys of each tile each and merge their softmax states at the end.
//   * Larger items (prefill chunks, shared-prefix groups): each warp owns 16
//     rows and takes every key.
// fp8 K/V are widened to f16 in registers (exact); the per-(layer, head) K
// scale is folded into the score scale and the V scale into the output.
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_args.h"
#include "attn_tile.cuh"
#include "common.cuh"
#include "internal.h"

namespace pkv {

// Issue the cp.async copies of key tile `tile` (keys k_begin + 64*tile ...) into ring slot `slot`.
template <int D, int KV, bool QBF>
PKV_DEVICE void load_tile(const AttnArgs& a, const PkvItem& it, const int32_t* bt_row, uint32_t sbase, int tile,
                          int slot, int tid) {
  using C = Cfg<D, KV, QBF>;
  constexpr int ROWS_PER_PASS = C::THREADS / C::CPR;
  const int ch = tid % C::CPR;
  const int r0 = tid / C::CPR;
  const int key0 = it.k_begin + tile * PKV_TILE_KEYS;
  const uint32_t kdst = sbase + slot * C::STAGE_BYTES;
  const int bmask = (1 << a.log2_block) - 1;
  const int64_t head_rows = int64_t(a.hkv) << a.log2_block;  // rows between K and V of a block
#pragma unroll
  for (int pass = 0; pass < PKV_TILE_KEYS / ROWS_PER_PASS; ++pass) {
    const int r = r0 + pass * ROWS_PER_PASS;
    const int kabs = key0 + r;
    const char* srck = static_cast<const char*>(a.pool);
    const char* srcv = srck;
    int bytes = 0;
    if (kabs < it.k_end) {
      const int phys = __ldg(bt_row + (kabs >> a.log2_block));
      if (phys >= 0 && phys < a.num_blocks) {
        const int64_t rowk = ((int64_t(phys) * a.num_layers + a.layer) * 2 * a.hkv + it.kv_head) * (int64_t(1) << a.log2_block) +
                             (kabs & bmask);
        srck += rowk * C::RB + ch * 16;
        srcv = srck + head_rows * C::RB;
        bytes = 16;
      } else if (ch == 0) {
        report(a.status, PKV_DEV_BAD_BLOCK_ID);
      }
    }
    const uint32_t off = tile_offset<C::RB>(r, ch * 16);
    cp_async16(kdst + off, srck, bytes);
    cp_async16(kdst + C::TILE_BYTES + off, srcv, bytes);
  }
}

template <int D, int KV, bool QBF>
__global__ void __launch_bounds__(128, 2) attn_mma_kernel(const AttnArgs a) {
  using C = Cfg<D, KV, QBF>;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int s_item;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g4 = lane >> 2, t4 = lane & 3;
  const uint32_t sbase = smem_addr(smem);
  const int total_q = __ldg(a.cu_q_lens + a.num_seqs);

  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(a.counter, 1u));
    __syncthreads();
    const int idx = s_item;
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
      __syncthreads();
      continue;
    }
    ItemCtx<D, KV, QBF> c;
    c.g = a.g;
    c.R = it.n_q * a.g;
    const bool decode = c.R <= 16;
    c.row_base = decode ? 0 : 16 * warp;
    const bool active = decode || c.row_base < c.R;
    load_q<D, KV, QBF>(a, it, c, g4, t4);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = c.row_base + g4 + 8 * hh;
      c.lim[hh] = (it.pos0 >= 0 && r < c.R) ? min(it.k_end, it.pos0 + r / c.g + 1) : it.k_end;
      c.lo[hh] = window_start(a.window, (it.pos0 >= 0 && r < c.R) ? it.pos0 + r / c.g : -1);
      c.m[hh] = -INFINITY;
      c.l[hh] = 0.f;
    }
#pragma unroll
    for (int nt = 0; nt < C::NNT; ++nt) c.acc[nt][0] = c.acc[nt][1] = c.acc[nt][2] = c.acc[nt][3] = 0.f;
    float scale_log2 = a.softmax_scale * kLog2e;
    float vscale = 1.f;
    if constexpr (KV == KV_E4M3) {
      scale_log2 *= __ldg(a.k_scale + a.layer * a.hkv + it.kv_head);
      vscale = __ldg(a.v_scale + a.layer * a.hkv + it.kv_head);
    }
    const int32_t* bt_row = a.block_tables + int64_t(it.seq) * a.max_blocks;
    const int ntiles = (it.k_end - it.k_begin + PKV_TILE_KEYS - 1) / PKV_TILE_KEYS;

#pragma unroll
    for (int i = 0; i < C::NST - 1; ++i) {
      if (i < ntiles) load_tile<D, KV, QBF>(a, it, bt_row, sbase, i, i, tid);
      cp_async_commit();
    }
    for (int i = 0; i < ntiles; ++i) {
      cp_async_wait<C::NST - 2>();
      __syncthreads();
      const int j = i + C::NST - 1;
      if (j < ntiles) load_tile<D, KV, QBF>(a, it, bt_row, sbase, j, j % C::NST, tid);
      cp_async_commit();
      const uint32_t kb = sbase + (i % C::NST) * C::STAGE_BYTES;
      const uint32_t vb = kb + C::TILE_BYTES;
      const int key0 = it.k_begin + i * PKV_TILE_KEYS;
      if (decode) {
        if (key0 + 16 * warp < it.k_end)
          compute_keys<1, D, KV, QBF>(a, c, kb, vb, 16 * warp, key0, g4, t4, lane, scale_log2);
      } else if (active) {
        compute_keys<4, D, KV, QBF>(a, c, kb, vb, 0, key0, g4, t4, lane, scale_log2);
      }
    }
    cp_async_wait<0>();
    __syncthreads();

    // Row sums over the quad.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      c.l[hh] += __shfl_xor_sync(0xffffffffu, c.l[hh], 1);
      c.l[hh] += __shfl_xor_sync(0xffffffffu, c.l[hh], 2);
    }
    const bool to_part = it.part_row >= 0;
    if (!decode) {
      if (active) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = c.row_base + g4 + 8 * hh;
          if (r >= c.R) continue;
          const float inv = c.l[hh] > 0.f ? vscale / c.l[hh] : 0.f;
          const float lse = c.l[hh] > 0.f ? (c.m[hh] + __log2f(c.l[hh])) * kLn2 : -INFINITY;
          const int64_t orow = to_part ? int64_t(it.part_row) + r
                                       : (int64_t(it.q_begin) + r / c.g) * a.hq + it.kv_head * c.g + r % c.g;
#pragma unroll
          for (int nt = 0; nt < C::NNT; ++nt)
#pragma unroll
            for (int e = 2 * hh; e < 2 * hh + 2; ++e) {
              const int d = acc_dim<KV>(nt, e, t4);
              const float v = c.acc[nt][e] * inv;
              if (to_part) a.part_o[orow * D + d] = v;
              else store_q_dtype<QBF>(a.out, orow * D + d, v);
            }
          if (t4 == 0) {
            if (to_part) a.part_lse[orow] = lse;
            else if (a.out_lse) a.out_lse[orow] = lse;
          }
        }
      }
    } else {
      // Merge the four warps' states through shared memory (the ring is idle now).
      float* red_o = reinterpret_cast<float*>(smem);          // [4][16][D]
      float* red_m = red_o + 4 * 16 * D;                      // [4][16]
      float* red_l = red_m + 4 * 16;                          // [4][16]
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = g4 + 8 * hh;
        if (r >= c.R) continue;
#pragma unroll
        for (int nt = 0; nt < C::NNT; ++nt)
#pragma unroll
          for (int e = 2 * hh; e < 2 * hh + 2; ++e) red_o[(warp * 16 + r) * D + acc_dim<KV>(nt, e, t4)] = c.acc[nt][e];
        if (t4 == 0) {
          red_m[warp * 16 + r] = c.m[hh];
          red_l[warp * 16 + r] = c.l[hh];
        }
      }
      __syncthreads();
      for (int x = tid; x < c.R * D; x += C::THREADS) {
        const int r = x / D, d = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * 16 + r]);
        float o = 0.f, lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float f = fast_exp2(red_m[w * 16 + r] - M);
            lsum += red_l[w * 16 + r] * f;
            o += red_o[(w * 16 + r) * D + d] * f;
          }
        }
        const float inv = lsum > 0.f ? vscale / lsum : 0.f;
        const int64_t orow = to_part ? int64_t(it.part_row) + r
                                     : (int64_t(it.q_begin) + r / c.g) * a.hq + it.kv_head * c.g + r % c.g;
        if (to_part) a.part_o[orow * D + d] = o * inv;
        else store_q_dtype<QBF>(a.out, orow * D + d, o * inv);
        if (d == 0) {
          const float lse = lsum > 0.f ? (M + __log2f(lsum)) * kLn2 : -INFINITY;
          if (to_part) a.part_lse[orow] = lse;
          else if (a.out_lse) a.out_lse[orow] = lse;
        }
      }
    }
    __syncthreads();
  }
}

template <int D, int KV, bool QBF>
cudaError_t launch_mma(const AttnArgs& a, int grid, cudaStream_t st) {
  attn_mma_kernel<D, KV, QBF><<<grid, Cfg<D, KV, QBF>::THREADS, Cfg<D, KV, QBF>::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D, int KV, bool QBF>
AttnKernel mma_kernel() {
  using C = Cfg<D, KV, QBF>;
  return AttnKernel{reinterpret_cast<const void*>(&attn_mma_kernel<D, KV, QBF>), C::THREADS, C::SMEM,
                    &launch_mma<D, KV, QBF>, PKV_TILE_ROWS};
}

AttnKernel f32_kernel(int head_dim);  // attn_f32.cu

bool attn_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k) {
  if (head_dim != 64 && head_dim != 128) return false;
  if (attn_tma_kernel_for(kv_dtype, q_dtype, head_dim, block_size, k)) return true;
  const bool d128 = head_dim == 128;
  switch (kv_dtype) {
    case PKV_F32:
      if (q_dtype != PKV_F32) return false;
      *k = f32_kernel(head_dim);
      return true;
    case PKV_BF16:
      if (q_dtype != PKV_BF16) return false;
      *k = d128 ? mma_kernel<128, KV_BF16, true>() : mma_kernel<64, KV_BF16, true>();
      return true;
    case PKV_F16:
      if (q_dtype != PKV_F16) return false;
      *k = d128 ? mma_kernel<128, KV_F16, false>() : mma_kernel<64, KV_F16, false>();
      return true;
    case PKV_FP8_E4M3:
      if (q_dtype == PKV_BF16) *k = d128 ? mma_kernel<128, KV_E4M3, true>() : mma_kernel<64, KV_E4M3, true>();
      else if (q_dtype == PKV_F16) *k = d128 ? mma_kernel<128, KV_E4M3, false>() : mma_kernel<64, KV_E4M3, false>();
      else return false;
      return true;
  }
  return false;
}

}  // namespace pkv
