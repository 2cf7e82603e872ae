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
#include "common.cuh"
#include "internal.h"

namespace pkv {

template <int D, int KV, bool QBF>
struct Cfg {
  static constexpr int ELEM = KV == KV_E4M3 ? 1 : 2;
  static constexpr int RB = D * ELEM;                    // bytes per K or V row
  static constexpr int TILE_BYTES = PKV_TILE_KEYS * RB;  // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NST = std::min(8, (96 * 1024) / STAGE_BYTES);
  static constexpr int SMEM = NST * STAGE_BYTES;
  static constexpr bool MMA_BF = KV == KV_BF16;
  static constexpr int NKS = D / 16;  // k-steps over the head dimension
  static constexpr int NNT = D / 8;   // n-tiles over the head dimension
  static constexpr int CPR = RB / 16; // 16-byte chunks per row
  static constexpr int THREADS = 128;
  static_assert(NST >= 2, "at least double buffering");
  static_assert(SMEM >= 4 * 16 * D * 4 + 2 * 64 * 4, "decode merge buffer fits in the stage ring");
};

// ---- per-item state and steps -------------------------------------------

template <int D, int KV, bool QBF>
struct ItemCtx {
  using C = Cfg<D, KV, QBF>;
  int R, row_base, g;
  int lim[2];          // exclusive key bound of rows g4 and g4 + 8
  float m[2], l[2];    // running max (log2 domain) and partial sum per row
  float acc[C::NNT][4];
  uint32_t qf[C::NKS][4];
};

// Load the warp's 16 query rows as A fragments, with the head dimension
// permuted so that thread t4 of a quad owns 16 consecutive dims per 64-dim
// group (matching the K fragments read with one 16-byte shared load).
template <int D, int KV, bool QBF>
PKV_DEVICE void load_q(const AttnArgs& a, const PkvItem& it, ItemCtx<D, KV, QBF>& c, int g4, int t4) {
  using C = Cfg<D, KV, QBF>;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = c.row_base + g4 + 8 * hh;
    const bool valid = r < c.R;
    const int64_t token = it.q_begin + (valid ? r / c.g : 0);
    const int head = it.kv_head * c.g + (valid ? r % c.g : 0);
    const uint16_t* qrow = static_cast<const uint16_t*>(a.q) + (token * a.hq + head) * D;
#pragma unroll
    for (int G = 0; G < D / 64; ++G) {
      uint32_t w[8];
      if (valid) {
        const uint4 x0 = *reinterpret_cast<const uint4*>(qrow + 64 * G + 16 * t4);
        const uint4 x1 = *reinterpret_cast<const uint4*>(qrow + 64 * G + 16 * t4 + 8);
        w[0] = x0.x; w[1] = x0.y; w[2] = x0.z; w[3] = x0.w; w[4] = x1.x; w[5] = x1.y; w[6] = x1.z; w[7] = x1.w;
        if constexpr (!C::MMA_BF && QBF) {  // bf16 query feeding f16 MMAs (fp8 pools)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = pack_f16x2(bf16_bits_to_float(uint16_t(w[i] & 0xffff)), bf16_bits_to_float(uint16_t(w[i] >> 16)));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = 0;
      }
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {
        c.qf[4 * G + s4][hh] = w[2 * s4];          // a0 / a1: dims 4*s4 + {0,1}
        c.qf[4 * G + s4][2 + hh] = w[2 * s4 + 1];  // a2 / a3: dims 4*s4 + {2,3}
      }
    }
  }
}

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

// One step over NSUB consecutive 16-key groups of a tile, starting at tile row kt0.
template <int NSUB, int D, int KV, bool QBF>
PKV_DEVICE void compute_keys(const AttnArgs& a, ItemCtx<D, KV, QBF>& c, uint32_t kbase, uint32_t vbase, int kt0,
                             int key0, int g4, int t4, int lane, float scale_log2) {
  using C = Cfg<D, KV, QBF>;
  float s[2 * NSUB][4];
#pragma unroll
  for (int nt = 0; nt < 2 * NSUB; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    const int kr = kt0 + 8 * nt + g4;
#pragma unroll
    for (int G = 0; G < D / 64; ++G) {
      if constexpr (KV == KV_E4M3) {
        const uint4 w = lds128(kbase + tile_offset<C::RB>(kr, 64 * G + 16 * t4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4)
          mma16816<false>(s[nt], c.qf[4 * G + s4], e4m3x2_to_f16x2(uint16_t(ww[s4] & 0xffff)),
                          e4m3x2_to_f16x2(uint16_t(ww[s4] >> 16)));
      } else {
        const uint4 w0 = lds128(kbase + tile_offset<C::RB>(kr, 2 * (64 * G + 16 * t4)));
        const uint4 w1 = lds128(kbase + tile_offset<C::RB>(kr, 2 * (64 * G + 16 * t4) + 16));
        const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) mma16816<C::MMA_BF>(s[nt], c.qf[4 * G + s4], ww[2 * s4], ww[2 * s4 + 1]);
      }
    }
  }
  // Scale, mask, online softmax (rows g4 and g4 + 8 of the warp's tile).
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2 * NSUB; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hh = e >> 1;
      const int key = key0 + kt0 + 8 * nt + 2 * t4 + (e & 1);
      const float v = key < c.lim[hh] ? s[nt][e] * scale_log2 : -INFINITY;
      s[nt][e] = v;
      mx[hh] = fmaxf(mx[hh], v);
    }
  float alpha[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
    mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
    const float mnew = fmaxf(c.m[hh], mx[hh]);
    const float muse = mnew == -INFINITY ? 0.f : mnew;
    alpha[hh] = fast_exp2(c.m[hh] - muse);
    c.m[hh] = mnew;
    mx[hh] = muse;
  }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2 * NSUB; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = fast_exp2(s[nt][e] - mx[e >> 1]);
      s[nt][e] = p;
      rs[e >> 1] += p;
    }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) c.l[hh] = c.l[hh] * alpha[hh] + rs[hh];
#pragma unroll
  for (int nt = 0; nt < C::NNT; ++nt) {
    c.acc[nt][0] *= alpha[0]; c.acc[nt][1] *= alpha[0];
    c.acc[nt][2] *= alpha[1]; c.acc[nt][3] *= alpha[1];
  }
  // P V.
#pragma unroll
  for (int kk = 0; kk < NSUB; ++kk) {
    uint32_t pa[4];
    if constexpr (C::MMA_BF) {
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    } else {
      pa[0] = pack_f16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_f16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_f16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_f16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    }
    const int vr = kt0 + 16 * kk + ((lane >> 3) & 1) * 8 + (lane & 7);
    if constexpr (KV == KV_E4M3) {
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vbase + tile_offset<C::RB>(vr, 32 * c32 + (lane >> 4) * 16), r0, r1, r2, r3);
        const uint32_t lo[2] = {__byte_perm(r0, 0, 0x3120), __byte_perm(r2, 0, 0x3120)};
        const uint32_t hi[2] = {__byte_perm(r1, 0, 0x3120), __byte_perm(r3, 0, 0x3120)};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c16 = 2 * c32 + half;
          mma16816<false>(c.acc[2 * c16], pa, e4m3x2_to_f16x2(uint16_t(lo[half] & 0xffff)),
                          e4m3x2_to_f16x2(uint16_t(hi[half] & 0xffff)));
          mma16816<false>(c.acc[2 * c16 + 1], pa, e4m3x2_to_f16x2(uint16_t(lo[half] >> 16)),
                          e4m3x2_to_f16x2(uint16_t(hi[half] >> 16)));
        }
      }
    } else {
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vbase + tile_offset<C::RB>(vr, 2 * (16 * dn + (lane >> 4) * 8)), r0, r1, r2, r3);
        mma16816<C::MMA_BF>(c.acc[2 * dn], pa, r0, r1);
        mma16816<C::MMA_BF>(c.acc[2 * dn + 1], pa, r2, r3);
      }
    }
  }
}

// Head-dimension index of accumulator element (nt, e) held by thread t4.
template <int KV>
PKV_DEVICE int acc_dim(int nt, int e, int t4) {
  if constexpr (KV == KV_E4M3) return 16 * (nt >> 1) + 4 * t4 + 2 * (e & 1) + (nt & 1);
  else return 8 * nt + 2 * t4 + (e & 1);
}

template <bool QBF, bool F32OUT = false>
PKV_DEVICE void store_q_dtype(void* out, int64_t idx, float v) {
  if constexpr (QBF) static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(out)[idx] = __float2half_rn(v);
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
              it.n_q * a.g <= PKV_TILE_ROWS && it.q_begin >= 0 && it.q_begin + it.n_q <= total_q && it.k_begin >= 0 &&
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
void launch_mma(const AttnArgs& a, int grid, cudaStream_t st) {
  attn_mma_kernel<D, KV, QBF><<<grid, Cfg<D, KV, QBF>::THREADS, Cfg<D, KV, QBF>::SMEM, st>>>(a);
}

template <int D, int KV, bool QBF>
AttnKernel mma_kernel() {
  using C = Cfg<D, KV, QBF>;
  return AttnKernel{reinterpret_cast<const void*>(&attn_mma_kernel<D, KV, QBF>), C::THREADS, C::SMEM,
                    &launch_mma<D, KV, QBF>};
}

AttnKernel f32_kernel(int head_dim);  // attn_f32.cu

bool attn_kernel_for(int kv_dtype, int q_dtype, int head_dim, AttnKernel* k) {
  if (head_dim != 64 && head_dim != 128) return false;
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
