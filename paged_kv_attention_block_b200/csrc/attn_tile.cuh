// Tile-level pieces shared by the attention kernels: shared-memory layout
// constants, query fragment loads, the row-split QK^T / online softmax / PV step
// on one staged K/V tile, and output index helpers.
#pragma once
#include <algorithm>

#include "attn_args.h"
#include "common.cuh"

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
  int lo[2];           // first key of rows g4 and g4 + 8 (limited attention window)
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

// One step over NSUB consecutive 16-key groups of a tile, starting at tile row kt0.
template <int NSUB, int D, int KV, bool QBF, int TK = PKV_TILE_KEYS, int SLAB = TK * 128>
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
        const uint4 w = lds128(kbase + tile_offset<C::RB, TK, SLAB>(kr, 64 * G + 16 * t4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4)
          mma16816<false>(s[nt], c.qf[4 * G + s4], e4m3x2_to_f16x2(uint16_t(ww[s4] & 0xffff)),
                          e4m3x2_to_f16x2(uint16_t(ww[s4] >> 16)));
      } else {
        const uint4 w0 = lds128(kbase + tile_offset<C::RB, TK, SLAB>(kr, 2 * (64 * G + 16 * t4)));
        const uint4 w1 = lds128(kbase + tile_offset<C::RB, TK, SLAB>(kr, 2 * (64 * G + 16 * t4) + 16));
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
      const float v = (key < c.lim[hh] && key >= c.lo[hh]) ? s[nt][e] * scale_log2 : -INFINITY;
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
        ldmatrix_x4_trans(vbase + tile_offset<C::RB, TK, SLAB>(vr, 32 * c32 + (lane >> 4) * 16), r0, r1, r2, r3);
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
        ldmatrix_x4_trans(vbase + tile_offset<C::RB, TK, SLAB>(vr, 2 * (16 * dn + (lane >> 4) * 8)), r0, r1, r2, r3);
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

}  // namespace pkv
