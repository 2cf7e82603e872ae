// Paged attention, TMA-fed and warp-specialised (bf16 / f16 / fp8-e4m3 pools,
// block size >= 8, 128- or 256-byte K/V rows; NVFP4 pools, d 128, block size
// >= 16).
//
// Same work list and results as attn_mma.cu (deep dive, gentlecold.top: §2
// decode reads all history KV, §6 one launch for a packed mix of prefill and
// decode requests, §8 causal chunks, §9 block pool and block tables); the data
// movement and the decode arithmetic are reorganised for sm_100a:
//
//   * Two persistent CTAs per SM: warp 4 is the producer, warps 0-3 consume.
//     The producer pulls items from the atomic counter (one item ahead),
//     publishes each item in a 2-slot descriptor ring, and streams the item's
//     K/V tiles (TK keys: 32 for 256-byte rows, 64 for 128-byte rows) into an
//     NST-stage shared-memory ring with 5-D TMA loads, 128-byte swizzle,
//     completion counted on an mbarrier.  Block ids arrive 32 at a time through
//     shared memory; when a tile lies inside one pool block a single box covers
//     its K and V rows (they are neighbours on the pool's K|V axis).  The
//     producer runs ahead across item boundaries, so the HBM queue does not
//     drain between items.  No load uses cluster multicast.
//   * Decode items (<= 16 rows): one consumer warp owns a whole tile (tiles go
//     round-robin over the 4 warps by tile index) and computes S^T = K Q^T and
//     O^T = V^T P^T, so the keys fill the 16-row MMA dimension and the
//     query-head group (g = 4 or 8 rows) fills n = 8.  P^T reaches the second
//     MMA through movmatrix.  Fragment addresses are fixed per lane; masking
//     runs only on tiles that reach past a row's limit.  The four warps merge
//     their softmax states at the end of the item.
//   * Four-head plans: each decode item covers KV heads kv_head .. kv_head + 3
//     of one query tile and key range, and warp w runs head kv_head + w over
//     the whole range (tile t: key tile t / 4, head t % 4).  A warp then holds
//     its head's complete state: it normalises and writes its rows itself,
//     with no merge between warps and no end-of-item barrier; the producer
//     reads the item's fields and block ids once for four heads.
//   * Tiles of more than 16 rows (prefill chunks, shared-prefix group tiles) go to
//     the tcgen05 kernel of attn_tc.cu; this kernel takes decode-sized items only.
//   * fp8 and NVFP4 tiles widen to f16 in registers with integer operations
//     (exact; values times a power of two taken back in the score and output
//     scales).  NVFP4 tiles arrive as two TMA boxes, E2M1 codes (64-byte rows,
//     64-byte swizzle) and E4M3 block scales, and each E2M1 value is multiplied
//     by its block scale in f16 (exact) before the MMA.  deep dive §13 (NVFP4
//     KV cache).
//   * Keys past the item's end inside the last tile are masked; their V rows
//     are zeroed in shared memory before the P V product (0 * NaN would leak).
//   * Every wait on an mbarrier is bounded; on a timeout the CTA records
//     PKV_DEV_TIMEOUT, stops issuing work and waits (bounded) for the loads it
//     has in flight before exiting.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "attn_args.h"
#include "attn_tile.cuh"
#include "common.cuh"
#include "internal.h"

namespace pkv {

template <int D, int KV, bool QBF>
struct TmaCfg {
  using L = Cfg<D, KV, QBF>;
  static constexpr bool FP4 = KV == KV_NVFP4;
  static constexpr int ELEM = L::ELEM;
  // Bytes per K or V row (NVFP4: the packed codes; the block scales travel separately).
  static constexpr int RB = FP4 ? D / 2 : L::RB;
  // Keys per tile: 32 for 256-byte rows, 64 for 128- and 64-byte rows.
  static constexpr int TK = RB == 256 ? 32 : 64;
  static constexpr int HALVES = FP4 ? 1 : RB / 128;  // 128-byte column slabs per row
  // Stage layout: [slab][K|V][TK rows][128 B]; K tile at +0, V tile at +TK*128.  NVFP4:
  // K codes [TK][64 B] (64-byte swizzle), V codes, then K and V block scales [TK][D/16 B].
  static constexpr int SLAB = 2 * TK * 128;
  static constexpr int TILE_BYTES = TK * RB;
  static constexpr int V_OFF = FP4 ? TILE_BYTES : TK * 128;
  static constexpr int SCALE_ROW = FP4 ? D / 16 : 0;
  static constexpr int KS_OFF = 2 * TILE_BYTES;
  static constexpr int VS_OFF = KS_OFF + TK * SCALE_ROW;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + 2 * TK * SCALE_ROW;
  // A multiple of 4: decode tiles go round-robin to the 4 consumer warps by tile
  // index within the item, so within an item every tile that lands in a given
  // stage belongs to the same warp and the stage's phases are consumed in order;
  // across items, the end-of-item merge barrier orders them.  Four-head items have
  // no such barrier: every item has a multiple of 4 tiles, so the running tile
  // count q stays a multiple of 4 and warp w always takes the tiles q + w + 4k,
  // whose stages (q + w + 4k) mod NST no other warp uses.
  // Four 16 KB stages (64 KB) leave room for two CTAs per SM: twice the producers and consumer
  // warps of one large-ring CTA, which measured faster than a 12-stage ring with one CTA per SM.
  static constexpr int NST = FP4 ? 8 : 4 * std::max(1, std::min(12, (64 * 1024) / STAGE_BYTES) / 4);
  static constexpr int IR = 2;  // item descriptor slots, each with the item's query rows
  // Query rows of a decode item, staged in shared memory with the item's descriptor: at most 16
  // rows (8 for NVFP4) of D 16-bit values.
  static constexpr int QROWS = FP4 ? PKV_FP4_ROWS : PKV_DECODE_ROWS;
  static constexpr int QSLOT = QROWS * D * 2;
  static constexpr int QBUF_BYTES = IR * QSLOT;
  static constexpr int MERGE_BYTES = 4 * 16 * D * 4 + 2 * 4 * 16 * 4;
  // Four-head plans never merge warps' states: their query slots (four heads' rows, IR of them)
  // and each warp's output staging (PKV_HEADS4_ROWS rows of D floats, padded so that the rows
  // 2 t4 + b a store instruction touches fall in distinct banks) live in the merge region.
  static constexpr int Q4SLOT = 4 * PKV_HEADS4_ROWS * D * 2;
  static constexpr int OSTRIDE = D + 4;
  static constexpr int OWARP = PKV_HEADS4_ROWS * OSTRIDE * 4;
  static constexpr int BAR_BYTES = 8 * (2 * NST + 2 * IR + 1);
  static constexpr int DESC_BYTES = IR * 64;
  static constexpr int IDS_BYTES = 32 * 4;
  static constexpr int SMEM =
      1024 + NST * STAGE_BYTES + MERGE_BYTES + QBUF_BYTES + BAR_BYTES + DESC_BYTES + IDS_BYTES + 16;
  static constexpr int THREADS = 160;
  static_assert(RB == 128 || RB == 256 || (FP4 && D == 128), "TMA path takes 128- or 256-byte rows, or NVFP4 d 128");
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the swizzle atoms aligned");
  static_assert(NST % 4 == 0, "stage count must be a multiple of the consumer warp count");
  static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
  static_assert(MERGE_BYTES % 16 == 0 && QSLOT % 16 == 0, "query slots 16-byte aligned for bulk copies");
  static_assert(IR * Q4SLOT + 4 * OWARP <= MERGE_BYTES && OWARP % 16 == 0, "four-head slots fit the merge region");
};

struct ItemDesc {
  int seq, kv_head, q_begin, n_q, k_begin, k_end, pos0, part_row, ntiles, state;  // state: 0 run, 1 skip, 2 end
  int pad[6];
};
static_assert(sizeof(ItemDesc) == 64, "descriptor slot");

struct TmaArgs {
  AttnArgs a;
  int32_t box_rows;  // rows per TMA box: TK when a tile lies inside one block, else the block size
  int32_t merged;    // 1: one box covers the K and V rows of a tile
};

// ---- decode-mode per-warp state (S^T / O^T formulation) -------------------
template <int D, int KV, bool QBF, int NR>
struct DecState {
  float acc[NR][D / 16][4];  // O^T fragments: [row group][d m-tile][frag]
  float m[NR][2], l[NR][2];  // rows 2*t4 + b (+8*group); m in scaled-log2 units
  uint32_t qb[NR][D / 16][2];
  int lim[NR][2];
  int lo[NR][2];  // first visible key (limited attention window)
};

template <int KV>
PKV_DEVICE int dec_dim(int mt, int e, int g4) {
  if constexpr (KV == KV_E4M3) return 32 * (mt >> 1) + 2 * g4 + 16 * (e >> 1) + (mt & 1);
  else if constexpr (KV == KV_NVFP4) return 64 * (mt >> 2) + 32 * (e >> 1) + 4 * g4 + (mt & 3);
  else return 16 * mt + g4 + 8 * (e >> 1);
}

// The decode tiles of fp8 and NVFP4 pools hold values times 2^-8 (E4M3) or 2^-7 (E2M1 code
// times block scale): x times the power of two back (exact).
template <int KV>
PKV_DEVICE float deq_undo(float x) {
  if constexpr (KV == KV_E4M3) return x * 256.f;
  else if constexpr (KV == KV_NVFP4) return x * 128.f;
  else return x;
}

// NVFP4 rows are 64 bytes; TMA's 64-byte swizzle XORs address bits 7..8 into the
// 16-byte chunk index (bits 4..5), so the 8-row ldmatrix phases hit distinct banks.
PKV_DEVICE uint32_t sw64(int row, int byte) {
  const uint32_t lin = uint32_t(row) * 64 + uint32_t(byte);
  return lin ^ (((lin >> 7) & 3) << 4);
}

// Per-lane shared-memory offsets of the K (A operand) and V (A^T operand)
// fragments for rows 0..15 of a tile; rows 16 further down add 16 * 128 bytes
// (the swizzle phase repeats every 8 rows).
template <int D, int KV, bool QBF>
struct DecOffsets {
  static constexpr int N = KV == KV_NVFP4 ? 2 : (KV == KV_E4M3 ? D / 32 : D / 16);
  uint32_t k[N], v[N];
};

template <int D, int KV, bool QBF>
PKV_DEVICE void dec_offsets(DecOffsets<D, KV, QBF>& o, int lane) {
  using T = TmaCfg<D, KV, QBF>;
  const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int i = 0; i < DecOffsets<D, KV, QBF>::N; ++i) {
    if constexpr (KV == KV_NVFP4) {
      // Column pair i = 16-byte chunks 2i, 2i+1 (dims 64i .. 64i+63).  K: matrix mi holds rows
      // 8*(mi & 1) .. +7 of chunk 2i + (mi >> 1); V (transposed): keys 8*(mi >> 1) .. +7 of
      // chunk 2i + (mi & 1).
      o.k[i] = sw64((mi & 1) * 8 + r8, 16 * (2 * i + (mi >> 1)));
      o.v[i] = sw64((mi >> 1) * 8 + r8, 16 * (2 * i + (mi & 1)));
    } else if constexpr (KV == KV_E4M3) {
      o.k[i] = tile_offset<T::RB, T::TK, T::SLAB>((mi & 1) * 8 + r8, 32 * i + (mi >> 1) * 16);
      o.v[i] = tile_offset<T::RB, T::TK, T::SLAB>((mi >> 1) * 8 + r8, 32 * i + (mi & 1) * 16);
    } else {
      o.k[i] = tile_offset<T::RB, T::TK, T::SLAB>((mi & 1) * 8 + r8, 2 * (16 * i + (mi >> 1) * 8));
      o.v[i] = tile_offset<T::RB, T::TK, T::SLAB>((mi >> 1) * 8 + r8, 2 * (16 * i + (mi & 1) * 8));
    }
  }
}

// The query rows of a decode item from its shared-memory slot (row r = token r / g, head r % g of
// the item's KV head, D 16-bit values each), as the B fragments of S^T = K Q^T.
// w4 >= 0: a four-head slot, whose token i holds the 4 g rows of the item's four heads; the rows
// of head w4 are token r / g, slot row 4 g (r / g) + g w4 + r % g.
template <int D, int KV, bool QBF, int NR>
PKV_DEVICE void dec_load_q(const AttnArgs& a, uint32_t qslot, int R, DecState<D, KV, QBF, NR>& st, int g4, int t4,
                           int w4) {
  constexpr bool MMA_BF = KV == KV_BF16;
#pragma unroll
  for (int nr = 0; nr < NR; ++nr) {
    const int r = nr * 8 + g4;
    const bool valid = r < R;
    const int sr = w4 < 0 ? r : (r / a.g) * 4 * a.g + w4 * a.g + r % a.g;
    const uint32_t qrow = qslot + uint32_t(valid ? sr : 0) * D * 2;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t w0 = 0, w1 = 0;
      if (valid) {
        if constexpr (KV == KV_NVFP4) {
          // k-step 2c + h pairs dims (b + 2h, b + 2h + 4) and (b + 2h + 1, b + 2h + 5), b = 32c + 8 t4:
          // the nibble pairs (i, i + 4) of the lane's K word.
          const uint4 x = lds128(qrow + 2 * (32 * (ks >> 1) + 8 * t4));
          const uint32_t lo = (ks & 1) ? x.y : x.x, hi = (ks & 1) ? x.w : x.z;
          w0 = __byte_perm(lo, hi, 0x5410);
          w1 = __byte_perm(lo, hi, 0x7632);
        } else if constexpr (KV == KV_E4M3) {
          // dims 16 ks + 4 t4 + {0, 2} and + {1, 3}: the byte pairs (0, 2), (1, 3) of the K word.
          const uint2 x = lds64(qrow + 2 * (16 * ks + 4 * t4));
          w0 = __byte_perm(x.x, x.y, 0x5410);
          w1 = __byte_perm(x.x, x.y, 0x7632);
        } else {
          w0 = lds32(qrow + 2 * (16 * ks + 2 * t4));
          w1 = lds32(qrow + 2 * (16 * ks + 8 + 2 * t4));
        }
        if constexpr (!MMA_BF && QBF) {
          w0 = pack_f16x2(bf16_bits_to_float(uint16_t(w0 & 0xffff)), bf16_bits_to_float(uint16_t(w0 >> 16)));
          w1 = pack_f16x2(bf16_bits_to_float(uint16_t(w1 & 0xffff)), bf16_bits_to_float(uint16_t(w1 >> 16)));
        }
      }
      st.qb[nr][ks][0] = w0;
      st.qb[nr][ks][1] = w1;
    }
  }
}

// One tile owned by this warp: S^T = K Q^T, online softmax per query row, O^T += V^T P^T.
// `masked`: some key of the tile is at or past some row's limit.  ksc / vsc: the tile's K and
// V block scales (NVFP4 pools only).
template <int D, int KV, bool QBF, int NR>
PKV_DEVICE void dec_tile(DecState<D, KV, QBF, NR>& st, const DecOffsets<D, KV, QBF>& off, uint32_t kbase,
                         uint32_t vbase, uint32_t ksc, uint32_t vsc, int key0, int lane, float c, bool masked) {
  using T = TmaCfg<D, KV, QBF>;
  constexpr int NKT = T::TK / 16;
  constexpr bool MMA_BF = KV == KV_BF16;
  constexpr int ROW = KV == KV_NVFP4 ? 64 : 128;  // bytes between rows of a slab
  const int g4 = lane >> 2;
  float s[NR][NKT][4];
#pragma unroll
  for (int kt = 0; kt < NKT; ++kt) {
#pragma unroll
    for (int nr = 0; nr < NR; ++nr) s[nr][kt][0] = s[nr][kt][1] = s[nr][kt][2] = s[nr][kt][3] = 0.f;
    const uint32_t kb = kbase + kt * 16 * ROW;
    if constexpr (KV == KV_NVFP4) {
      // Block scales of keys g4 and g4 + 8 (eight bytes each: groups 0-3, 4-7); the lane's
      // eight dims of chunk c lie in group 2c + (t4 >> 1).
      const int t4 = lane & 3;
      const uint2 s0 = lds64(ksc + uint32_t(kt * 16 + g4) * 8);
      const uint2 s1 = lds64(ksc + uint32_t(kt * 16 + g4 + 8) * 8);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        uint32_t r[4];  // key g4 chunk 2p, key g4+8 chunk 2p, key g4 chunk 2p+1, key g4+8 chunk 2p+1
        ldmatrix_x4(kb + off.k[p], r[0], r[1], r[2], r[3]);
        const uint32_t w0 = p ? s0.y : s0.x, w1 = p ? s1.y : s1.x;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          // Block scale byte b of keys g4 and g4 + 8 into bytes 1 and 3, as f16x2 (s, s) * 2^7.
          const uint32_t b = uint32_t(2 * cc + (t4 >> 1));
          const uint32_t sel = (b << 4) | (b << 12);
          const uint32_t sg = hmul2(e4m3_b13_f16x2(__byte_perm(w0, 0, sel)), kF16Pow2_15x2);
          const uint32_t sg8 = hmul2(e4m3_b13_f16x2(__byte_perm(w1, 0, sel)), kF16Pow2_15x2);
          const uint32_t lo = r[2 * cc], hi = r[2 * cc + 1];
          // Nibble pairs (i, i+4) of each word as f16x2 values * 2^-14; times the scales: * 2^-7.
          const uint32_t l0 = hmul2(e2m1_pair_f16x2<0>(lo), sg), l1 = hmul2(e2m1_pair_f16x2<1>(lo), sg);
          const uint32_t l2 = hmul2(e2m1_pair_f16x2<2>(lo), sg), l3 = hmul2(e2m1_pair_f16x2<3>(lo), sg);
          const uint32_t h0 = hmul2(e2m1_pair_f16x2<0>(hi), sg8), h1 = hmul2(e2m1_pair_f16x2<1>(hi), sg8);
          const uint32_t h2 = hmul2(e2m1_pair_f16x2<2>(hi), sg8), h3 = hmul2(e2m1_pair_f16x2<3>(hi), sg8);
          // k-step 2c + h: k (2t, 2t+1) = dims (b + 2h, b + 2h + 4), (2t+8, 2t+9) = (b + 2h + 1, b + 2h + 5).
          const uint32_t k0[4] = {l0, h0, l1, h1}, k1[4] = {l2, h2, l3, h3};
          const int ks = 2 * (2 * p + cc);
#pragma unroll
          for (int nr = 0; nr < NR; ++nr) {
            mma16816<false>(s[nr][kt], k0, st.qb[nr][ks][0], st.qb[nr][ks][1]);
            mma16816<false>(s[nr][kt], k1, st.qb[nr][ks + 1][0], st.qb[nr][ks + 1][1]);
          }
        }
      }
    } else if constexpr (KV == KV_E4M3) {
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(kb + off.k[kp], r0, r1, r2, r3);
        // Values times 2^-8 (undone in the softmax scale).
        const uint32_t a0[4] = {e4m3_b02_f16x2(r0), e4m3_b02_f16x2(r1), e4m3_b13_f16x2(r0), e4m3_b13_f16x2(r1)};
        const uint32_t a1[4] = {e4m3_b02_f16x2(r2), e4m3_b02_f16x2(r3), e4m3_b13_f16x2(r2), e4m3_b13_f16x2(r3)};
#pragma unroll
        for (int nr = 0; nr < NR; ++nr) {
          mma16816<false>(s[nr][kt], a0, st.qb[nr][2 * kp][0], st.qb[nr][2 * kp][1]);
          mma16816<false>(s[nr][kt], a1, st.qb[nr][2 * kp + 1][0], st.qb[nr][2 * kp + 1][1]);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(kb + off.k[ks], a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nr = 0; nr < NR; ++nr) mma16816<MMA_BF>(s[nr][kt], a, st.qb[nr][ks][0], st.qb[nr][ks][1]);
      }
    }
  }
  if (masked) {
#pragma unroll
    for (int nr = 0; nr < NR; ++nr)
#pragma unroll
      for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
        {
          const int key = key0 + kt * 16 + g4 + 8 * (e >> 1);
          if (key >= st.lim[nr][e & 1] || key < st.lo[nr][e & 1]) s[nr][kt][e] = -INFINITY;
        }
  }
  // Running max per query row (in raw score units, then scaled), exp2 of the scaled scores.
#pragma unroll
  for (int nr = 0; nr < NR; ++nr) {
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
      for (int e = 0; e < 4; ++e) mx[e & 1] = fmaxf(mx[e & 1], s[nr][kt][e]);
    float alpha[2], mneg[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float x = mx[b];
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
      const float mnew = fmaxf(st.m[nr][b], x * c);
      const float muse = mnew == -INFINITY ? 0.f : mnew;
      alpha[b] = fast_exp2(st.m[nr][b] - muse);
      st.m[nr][b] = mnew;
      mneg[b] = -muse;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = fast_exp2(fmaf(s[nr][kt][e], c, mneg[e & 1]));
        s[nr][kt][e] = p;
        rs[e & 1] += p;
      }
    st.l[nr][0] = st.l[nr][0] * alpha[0] + rs[0];
    st.l[nr][1] = st.l[nr][1] * alpha[1] + rs[1];
    // Once the running maxima settle, most tiles leave every alpha at 1: skip the rescale then.
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.acc[nr][mt][0] *= alpha[0];
        st.acc[nr][mt][1] *= alpha[1];
        st.acc[nr][mt][2] *= alpha[0];
        st.acc[nr][mt][3] *= alpha[1];
      }
    }
  }
  // O^T += V^T P^T, 16 keys at a time.
#pragma unroll
  for (int kt = 0; kt < NKT; ++kt) {
    uint32_t pb[NR][2];
#pragma unroll
    for (int nr = 0; nr < NR; ++nr) {
      if constexpr (MMA_BF) {
        pb[nr][0] = movmatrix_trans(pack_bf16x2(s[nr][kt][0], s[nr][kt][1]));
        pb[nr][1] = movmatrix_trans(pack_bf16x2(s[nr][kt][2], s[nr][kt][3]));
      } else {
        pb[nr][0] = movmatrix_trans(pack_f16x2(s[nr][kt][0], s[nr][kt][1]));
        pb[nr][1] = movmatrix_trans(pack_f16x2(s[nr][kt][2], s[nr][kt][3]));
      }
    }
    const uint32_t vb = vbase + kt * 16 * ROW;
    if constexpr (KV == KV_NVFP4) {
      // V block scales of keys (2t4, 2t4+1) and (2t4+8, 2t4+9): two adjacent 8-byte rows each.
      // The lane's dims of chunk c lie in group 2c + (g4 >> 2).
      const int t4 = lane & 3;
      const uint4 v0 = lds128(vsc + uint32_t(kt * 16 + 2 * t4) * 8);
      const uint4 v1 = lds128(vsc + uint32_t(kt * 16 + 8 + 2 * t4) * 8);
      const uint32_t bA = uint32_t(g4 >> 2), bB = bA + 2;
      const uint32_t selA = (bA << 4) | ((bA + 4) << 12), selB = (bB << 4) | ((bB + 4) << 12);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        uint32_t x[4];  // keys 0-7 chunk 2p, keys 0-7 chunk 2p+1, keys 8-15 chunk 2p, keys 8-15 chunk 2p+1
        ldmatrix_x4_trans(vb + off.v[p], x[0], x[1], x[2], x[3]);
        const uint32_t a0w = p ? v0.y : v0.x, a1w = p ? v0.w : v0.z;  // keys 2t4, 2t4+1
        const uint32_t b0w = p ? v1.y : v1.x, b1w = p ? v1.w : v1.z;  // keys 2t4+8, 2t4+9
        // (key 2t, key 2t+1) scale pairs in bytes 1 and 3, as f16x2 * 2^7.
        const uint32_t sc[4] = {hmul2(e4m3_b13_f16x2(__byte_perm(a0w, a1w, selA)), kF16Pow2_15x2),
                                hmul2(e4m3_b13_f16x2(__byte_perm(a0w, a1w, selB)), kF16Pow2_15x2),
                                hmul2(e4m3_b13_f16x2(__byte_perm(b0w, b1w, selA)), kF16Pow2_15x2),
                                hmul2(e4m3_b13_f16x2(__byte_perm(b0w, b1w, selB)), kF16Pow2_15x2)};
        // Each word: key 2t's codes of dims 4 g4 + 0..3 (bits 0..15), key 2t+1's (bits 16..31): nibble
        // pair (i, i+4) is the key pair of dim 4 g4 + i, as f16x2 * 2^-14; times the scales: * 2^-7.
#define PKV_FP4_V_MTILE(I)                                                                                        \
  {                                                                                                               \
    const uint32_t a[4] = {hmul2(e2m1_pair_f16x2<I>(x[0]), sc[0]), hmul2(e2m1_pair_f16x2<I>(x[1]), sc[1]),       \
                           hmul2(e2m1_pair_f16x2<I>(x[2]), sc[2]), hmul2(e2m1_pair_f16x2<I>(x[3]), sc[3])};      \
    _Pragma("unroll") for (int nr = 0; nr < NR; ++nr) mma16816<false>(st.acc[nr][4 * p + I], a, pb[nr][0], pb[nr][1]); \
  }
        // m-tile 4p + i: rows g4 -> dim 64p + 4 g4 + i, rows g4 + 8 -> dim 64p + 32 + 4 g4 + i.
        PKV_FP4_V_MTILE(0)
        PKV_FP4_V_MTILE(1)
        PKV_FP4_V_MTILE(2)
        PKV_FP4_V_MTILE(3)
#undef PKV_FP4_V_MTILE
      }
    } else if constexpr (KV == KV_E4M3) {
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vb + off.v[c32], r0, r1, r2, r3);
        // Each word holds (key 2t: dims d, d+1)(key 2t+1: dims d, d+1): bytes (0, 2) are the key
        // pair of dim d, bytes (1, 3) of dim d+1.  Values times 2^-8 (undone in the output scale).
        const uint32_t ae[4] = {e4m3_b02_f16x2(r0), e4m3_b02_f16x2(r1), e4m3_b02_f16x2(r2), e4m3_b02_f16x2(r3)};
        const uint32_t ao[4] = {e4m3_b13_f16x2(r0), e4m3_b13_f16x2(r1), e4m3_b13_f16x2(r2), e4m3_b13_f16x2(r3)};
#pragma unroll
        for (int nr = 0; nr < NR; ++nr) {
          mma16816<false>(st.acc[nr][2 * c32], ae, pb[nr][0], pb[nr][1]);
          mma16816<false>(st.acc[nr][2 * c32 + 1], ao, pb[nr][0], pb[nr][1]);
        }
      }
    } else {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a[4];
        ldmatrix_x4_trans(vb + off.v[mt], a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nr = 0; nr < NR; ++nr) mma16816<MMA_BF>(st.acc[nr][mt], a, pb[nr][0], pb[nr][1]);
      }
    }
  }
}

// NVFP4 tile, 16 keys at a time: S^T for 16 keys, the online-softmax update, then O^T += V^T P^T
// for those keys.  The dequantisation roughly triples the instruction count of a tile, so the
// loop over the tile's 16-key steps is kept rolled: its body stays small enough for the
// instruction cache (a fully unrolled 64-key tile was stalled on instruction fetch).
template <int D, bool QBF>
PKV_DEVICE void dec_tile_fp4(DecState<D, KV_NVFP4, QBF, 1>& st, const DecOffsets<D, KV_NVFP4, QBF>& off, uint32_t kbase,
                             uint32_t vbase, uint32_t ksc, uint32_t vsc, int key0, int lane, float c, bool masked) {
  using T = TmaCfg<D, KV_NVFP4, QBF>;
  constexpr int NKT = T::TK / 16;
  constexpr int ROW = 64;  // bytes between rows of codes
  const int g4 = lane >> 2, t4 = lane & 3;
#pragma unroll 1
  for (int kt = 0; kt < NKT; ++kt) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kb = kbase + kt * 16 * ROW;
    {
      // Block scales of keys g4 and g4 + 8 (eight bytes each: groups 0-3, 4-7); the lane's eight
      // dims of chunk c lie in group 2c + (t4 >> 1).
      const uint2 s0 = lds64(ksc + uint32_t(kt * 16 + g4) * 8);
      const uint2 s1 = lds64(ksc + uint32_t(kt * 16 + g4 + 8) * 8);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        uint32_t r[4];  // key g4 chunk 2p, key g4+8 chunk 2p, key g4 chunk 2p+1, key g4+8 chunk 2p+1
        ldmatrix_x4(kb + off.k[p], r[0], r[1], r[2], r[3]);
        const uint32_t w0 = p ? s0.y : s0.x, w1 = p ? s1.y : s1.x;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          // Block scale byte b of keys g4 and g4 + 8 into bytes 1 and 3, as f16x2 (s, s) * 2^7.
          const uint32_t b = uint32_t(2 * cc + (t4 >> 1));
          const uint32_t sel = (b << 4) | (b << 12);
          const uint32_t sg = hmul2(e4m3_b13_f16x2(__byte_perm(w0, 0, sel)), kF16Pow2_15x2);
          const uint32_t sg8 = hmul2(e4m3_b13_f16x2(__byte_perm(w1, 0, sel)), kF16Pow2_15x2);
          uint32_t pl[4], ph[4];  // nibble pairs (i, i+4) of the lo and hi words
          e2m1_word_f16x2(r[2 * cc], pl);
          e2m1_word_f16x2(r[2 * cc + 1], ph);
          const uint32_t k0[4] = {hmul2(pl[0], sg), hmul2(ph[0], sg8), hmul2(pl[1], sg), hmul2(ph[1], sg8)};
          const uint32_t k1[4] = {hmul2(pl[2], sg), hmul2(ph[2], sg8), hmul2(pl[3], sg), hmul2(ph[3], sg8)};
          const int ks = 2 * (2 * p + cc);
          mma16816<false>(s4, k0, st.qb[0][ks][0], st.qb[0][ks][1]);
          mma16816<false>(s4, k1, st.qb[0][ks + 1][0], st.qb[0][ks + 1][1]);
        }
      }
    }
    if (masked) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + kt * 16 + g4 + 8 * (e >> 1);
        if (key >= st.lim[0][e & 1] || key < st.lo[0][e & 1]) s4[e] = -INFINITY;
      }
    }
    // Online softmax over these 16 keys for the lane's two query rows.
    float alpha[2], mneg[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float x = fmaxf(s4[b], s4[b + 2]);
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
      x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
      const float mnew = fmaxf(st.m[0][b], x * c);
      const float muse = mnew == -INFINITY ? 0.f : mnew;
      alpha[b] = fast_exp2(st.m[0][b] - muse);
      st.m[0][b] = mnew;
      mneg[b] = -muse;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s4[e] = fast_exp2(fmaf(s4[e], c, mneg[e & 1]));
      rs[e & 1] += s4[e];
    }
    st.l[0][0] = st.l[0][0] * alpha[0] + rs[0];
    st.l[0][1] = st.l[0][1] * alpha[1] + rs[1];
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.acc[0][mt][0] *= alpha[0];
        st.acc[0][mt][1] *= alpha[1];
        st.acc[0][mt][2] *= alpha[0];
        st.acc[0][mt][3] *= alpha[1];
      }
    }
    const uint32_t pb0 = movmatrix_trans(pack_f16x2(s4[0], s4[1]));
    const uint32_t pb1 = movmatrix_trans(pack_f16x2(s4[2], s4[3]));
    // O^T += V^T P^T for these keys.  V block scales of keys (2t4, 2t4+1) and (2t4+8, 2t4+9): two
    // adjacent 8-byte rows each; the lane's dims of chunk c lie in group 2c + (g4 >> 2).
    const uint32_t vb = vbase + kt * 16 * ROW;
    const uint4 v0 = lds128(vsc + uint32_t(kt * 16 + 2 * t4) * 8);
    const uint4 v1 = lds128(vsc + uint32_t(kt * 16 + 8 + 2 * t4) * 8);
    const uint32_t bA = uint32_t(g4 >> 2), bB = bA + 2;
    const uint32_t selA = (bA << 4) | ((bA + 4) << 12), selB = (bB << 4) | ((bB + 4) << 12);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      uint32_t x[4];  // keys 0-7 chunk 2p, keys 0-7 chunk 2p+1, keys 8-15 chunk 2p, keys 8-15 chunk 2p+1
      ldmatrix_x4_trans(vb + off.v[p], x[0], x[1], x[2], x[3]);
      const uint32_t a0w = p ? v0.y : v0.x, a1w = p ? v0.w : v0.z;  // keys 2t4, 2t4+1
      const uint32_t b0w = p ? v1.y : v1.x, b1w = p ? v1.w : v1.z;  // keys 2t4+8, 2t4+9
      // (key 2t, key 2t+1) scale pairs in bytes 1 and 3, as f16x2 * 2^7.
      const uint32_t sc[4] = {hmul2(e4m3_b13_f16x2(__byte_perm(a0w, a1w, selA)), kF16Pow2_15x2),
                              hmul2(e4m3_b13_f16x2(__byte_perm(a0w, a1w, selB)), kF16Pow2_15x2),
                              hmul2(e4m3_b13_f16x2(__byte_perm(b0w, b1w, selA)), kF16Pow2_15x2),
                              hmul2(e4m3_b13_f16x2(__byte_perm(b0w, b1w, selB)), kF16Pow2_15x2)};
      uint32_t px[4][4];  // word k's nibble pairs (i, i+4)
#pragma unroll
      for (int k = 0; k < 4; ++k) e2m1_word_f16x2(x[k], px[k]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // m-tile 4p + i: rows g4 -> dim 64p + 4 g4 + i, rows g4 + 8 -> dim 64p + 32 + 4 g4 + i.
        const uint32_t a[4] = {hmul2(px[0][i], sc[0]), hmul2(px[1][i], sc[1]), hmul2(px[2][i], sc[2]),
                               hmul2(px[3][i], sc[3])};
        mma16816<false>(st.acc[0][4 * p + i], a, pb0, pb1);
      }
    }
  }
}

// NVFP4: zero V code rows [from, TK) (64 bytes each; the swizzle only permutes chunks within a
// row) and their block scale rows (D/16 bytes each) of a staged tile.
template <int TK, int SROW>
PKV_DEVICE void zero_v_tail_fp4(uint32_t vbase, uint32_t vscale, int from, int lane) {
  for (int x = lane; x < (TK - from) * 4; x += 32)
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(vbase + uint32_t(from * 64 + x * 16)), "r"(0) : "memory");
  for (int x = lane; x < (TK - from) * SROW / 8; x += 32)
    asm volatile("st.shared.v2.u32 [%0], {%1,%1};\n" ::"r"(vscale + uint32_t(from * SROW + x * 8)), "r"(0) : "memory");
  __syncwarp();
}

// Zero V rows [from, TK) of a staged tile: those keys are past the item's end.
template <int RB, int TK, int SLAB>
PKV_DEVICE void zero_v_tail(uint32_t vbase, int from, int lane) {
  constexpr int CPR = RB / 16;
  for (int x = lane; x < (TK - from) * CPR; x += 32) {
    const int r = from + x / CPR, ch = x % CPR;
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(vbase + tile_offset<RB, TK, SLAB>(r, ch * 16)), "r"(0)
                 : "memory");
  }
  __syncwarp();
}

// Four-head items: one warp writes its head's R (<= 8) rows from its staging rows (row r: D
// unnormalised dims, then the row's max and sum in scaled-log2 units), TPR lanes a row and DPT
// consecutive dims each.  part_row >= 0: float32 partial rows part_row + r; else output rows of
// token q_begin + r / g, head head * g + r % g.
template <int D, int KV, bool QBF>
PKV_DEVICE void h4_write_rows(const float* ob, int R, int lane, int g, int hq, int q_begin, int head,
                                           int part_row, float vscale, void* out, float* out_lse, float* part_o,
                                           float* part_lse) {
  using T = TmaCfg<D, KV, QBF>;
  const int Rp = R <= 4 ? 4 : 8;
  const int TPR = 32 / Rp, DPT = D / TPR;
  const int r = lane / TPR, d0 = (lane % TPR) * DPT;
  if (r >= R) return;
  const float M = ob[r * T::OSTRIDE + D], lsum = ob[r * T::OSTRIDE + D + 1];
  const float inv = lsum > 0.f ? vscale / lsum : 0.f;
  const float lse2 = lsum > 0.f ? M + __log2f(lsum) : -INFINITY;
  const bool to_part = part_row >= 0;
  const int64_t orow = to_part ? int64_t(part_row) + r : (int64_t(q_begin) + r / g) * hq + head * g + r % g;
#pragma unroll 1
  for (int c = 0; c < DPT; c += 4) {
    float4 o = *reinterpret_cast<const float4*>(ob + r * T::OSTRIDE + d0 + c);
    o.x *= inv;
    o.y *= inv;
    o.z *= inv;
    o.w *= inv;
    if (to_part) {
      *reinterpret_cast<float4*>(part_o + orow * D + d0 + c) = o;
    } else {
      const uint2 pk = QBF ? make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w))
                           : make_uint2(pack_f16x2(o.x, o.y), pack_f16x2(o.z, o.w));
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + orow * D + d0 + c) = pk;
    }
  }
  if (lane % TPR == 0) {
    const float lse = lse2 * kLn2;
    if (to_part) part_lse[orow] = lse;
    else if (out_lse) out_lse[orow] = lse;
  }
}

// H4: the four-head variant, launched for plans whose decode items cover four KV heads each.
template <int D, int KV, bool QBF, bool H4>
__global__ void __launch_bounds__(160, 2) attn_tma_kernel(const __grid_constant__ CUtensorMap tmap,
                                                          const __grid_constant__ CUtensorMap smap, const TmaArgs ta) {
  using T = TmaCfg<D, KV, QBF>;
  const AttnArgs& a = ta.a;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t stages = base;
  float* red_o = reinterpret_cast<float*>(base_ptr + T::NST * T::STAGE_BYTES);
  float* red_m = red_o + 4 * 16 * D;
  float* red_l = red_m + 4 * 16;
  const uint32_t qbuf = base + T::NST * T::STAGE_BYTES + T::MERGE_BYTES;  // T::IR query slots
  // Four-head plans: T::IR query slots at the start of the merge region, the warps' output
  // staging after them.
  const uint32_t q4buf = base + T::NST * T::STAGE_BYTES;
  constexpr bool h4 = H4;  // every decode item covers four KV heads
  const uint32_t bars = qbuf + T::QBUF_BYTES;
  auto full_bar = [&](int i) { return bars + 8 * i; };
  auto empty_bar = [&](int i) { return bars + 8 * (T::NST + i); };
  auto ifull_bar = [&](int i) { return bars + 8 * (2 * T::NST + i); };
  auto iempty_bar = [&](int i) { return bars + 8 * (2 * T::NST + T::IR + i); };
  const uint32_t merge_bar = bars + 8 * (2 * T::NST + 2 * T::IR);
  ItemDesc* descs =
      reinterpret_cast<ItemDesc*>(base_ptr + T::NST * T::STAGE_BYTES + T::MERGE_BYTES + T::QBUF_BYTES + T::BAR_BYTES);
  volatile int* s_ids = reinterpret_cast<volatile int*>(base_ptr + T::NST * T::STAGE_BYTES + T::MERGE_BYTES +
                                                        T::QBUF_BYTES + T::BAR_BYTES + T::DESC_BYTES);
  __shared__ volatile int s_abort;
  __shared__ long long s_wl;  // SM cycles any one wait may take

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < T::NST; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 4);
    }
    for (int i = 0; i < T::IR; ++i) {
      mbar_init(ifull_bar(i), 1);
      mbar_init(iempty_bar(i), 4);
    }
    mbar_init(merge_bar, 128);
    s_abort = 0;
    s_wl = a.wait_limit;
    fence_mbar_init();
  }
  // First: launched as a programmatic dependent of the plan staging, the barriers above are set
  // up while that runs; nothing it or the work before it wrote (the plan, the appended K/V, q)
  // is read before this.  A no-op when the kernel ahead is not a programmatic primary.  Second
  // (beside the tcgen05 kernel): that kernel waited for the plan staging before it let this
  // launch.
  if (a.pdl_role == 0) pdl_wait();
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // The warp fetches item fields and 32 block ids at a time (coalesced);
    // lane 0 alone runs the tile loop: wait for a free stage, arm its barrier,
    // issue the boxes.
    const int total_q = __ldg(a.cu_q_lens + a.num_seqs);
    const int box_rows = ta.box_rows;
    const bool merged = ta.merged != 0;
    const int bmask = (1 << a.log2_block) - 1;
    const int c3k = 2 * a.layer;
    int q = 0, it_seq = 0;
    bool ok = true;
    // The first item of each CTA is its own index; later ones come from the counter.
    int next_idx = blockIdx.x;
    for (;;) {
      const int slot = it_seq % T::IR;
      int flag = 1;
      if (lane == 0) flag = mbar_wait(iempty_bar(slot), ((it_seq / T::IR) & 1) ^ 1, &s_wl) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, flag, 0)) { ok = false; break; }
      const int idx = __shfl_sync(0xffffffffu, next_idx, 0);
      ItemDesc& d = descs[slot];
      if (idx >= a.n_items) {
        if (lane == 0) {
          d.state = 2;
          mbar_arrive(ifull_bar(slot), 1);
        }
        break;
      }
      if (lane == 0) next_idx = int(gridDim.x + atomicAdd(a.counter, 1u));  // the next item, fetched ahead
      const int* src = reinterpret_cast<const int*>(a.items + idx);
      const int field = lane < 8 ? __ldg(src + lane) : 0;
      PkvItem it;
      it.seq = __shfl_sync(0xffffffffu, field, 0);
      it.kv_head = __shfl_sync(0xffffffffu, field, 1);
      it.q_begin = __shfl_sync(0xffffffffu, field, 2);
      it.n_q = __shfl_sync(0xffffffffu, field, 3);
      it.k_begin = __shfl_sync(0xffffffffu, field, 4);
      it.k_end = __shfl_sync(0xffffffffu, field, 5);
      it.pos0 = __shfl_sync(0xffffffffu, field, 6);
      it.part_row = __shfl_sync(0xffffffffu, field, 7);
      bool valid = it.seq >= 0 && it.seq < a.num_seqs && it.kv_head >= 0 && it.kv_head < a.hkv && it.n_q > 0 &&
                   it.n_q * a.g <= a.max_rows && it.q_begin >= 0 && it.q_begin + it.n_q <= total_q &&
                   it.k_begin >= 0 && it.k_begin < it.k_end && (it.k_begin % box_rows) == 0 &&
                   (!h4 || (it.kv_head % 4 == 0 && it.kv_head + 4 <= a.hkv && it.n_q * a.g <= PKV_HEADS4_ROWS));
      if (valid) {
        const int L = __ldg(a.seq_lens + it.seq);
        valid = it.k_end <= L && ((it.k_end - 1) >> a.log2_block) < a.max_blocks && (it.pos0 < 0 || it.pos0 + it.n_q <= L);
      }
      if (!valid && lane == 0) report(a.status, PKV_DEV_PLAN_MISMATCH);
      // Four-head items: 4 tiles per key tile, tile t of head kv_head + t % 4.
      const int ntiles = valid ? ((it.k_end - it.k_begin + T::TK - 1) / T::TK) * (h4 ? 4 : 1) : 0;
      if (lane == 0) {
        d.seq = it.seq; d.kv_head = it.kv_head; d.q_begin = it.q_begin; d.n_q = it.n_q; d.k_begin = it.k_begin;
        d.k_end = it.k_end; d.pos0 = it.pos0; d.part_row = it.part_row; d.ntiles = ntiles; d.state = valid ? 0 : 1;
        const int rows = it.n_q * a.g;
        if (valid && rows <= T::QROWS) {
          // A decode item's query rows travel with its descriptor: for each of its tokens the g
          // heads of the KV head (4 g of the four KV heads) are one contiguous run of 16-bit
          // values; the slot's barrier completes when they have landed.
          const uint32_t run = uint32_t(a.g) * D * 2 * (h4 ? 4u : 1u);
          const uint32_t qdst = h4 ? q4buf + slot * T::Q4SLOT : qbuf + slot * T::QSLOT;
          mbar_arrive_expect_tx(ifull_bar(slot), run * uint32_t(it.n_q));
          const uint16_t* qsrc = static_cast<const uint16_t*>(a.q) + (int64_t(it.q_begin) * a.hq + it.kv_head * a.g) * D;
          for (int i = 0; i < it.n_q; ++i)
            bulk_load_1d(qdst + uint32_t(i) * run, qsrc + int64_t(i) * a.hq * D, run, ifull_bar(slot));
        } else {
          mbar_arrive(ifull_bar(slot), 1);
        }
      }
      ++it_seq;
      if (ntiles == 0) continue;
      // Test switch: publish the item but load none of its tiles, so every consumer wait runs out.
      if (a.debug_flags & PKV_DEBUG_WITHHOLD_LOADS) continue;
      const int32_t* bt_row = a.block_tables + int64_t(it.seq) * a.max_blocks;
      const int first_blk = it.k_begin >> a.log2_block;
      const int nblk_item = ((it.k_end - 1) >> a.log2_block) - first_blk + 1;
      int t = 0;
      for (int chunk = 0; chunk < nblk_item && ok; chunk += 32) {
        s_ids[lane] = chunk + lane < nblk_item ? __ldg(bt_row + first_blk + chunk + lane) : -1;
        __syncwarp();
        if (lane == 0) {
          // Tiles whose first block lies in this chunk (a tile never straddles chunks:
          // 32 is a multiple of the blocks per tile).
          for (; t < ntiles; ++t, ++q) {
            const int key0 = it.k_begin + (h4 ? t >> 2 : t) * T::TK;
            const int head = it.kv_head + (h4 ? t & 3 : 0);
            const int rel = (key0 >> a.log2_block) - first_blk - chunk;
            if (rel >= 32) break;
            const int stg = q % T::NST;
            if (s_abort || !mbar_wait(empty_bar(stg), ((q / T::NST) & 1) ^ 1, &s_wl)) { flag = 0; break; }
            const uint32_t sdst = stages + stg * T::STAGE_BYTES;
            if constexpr (T::FP4) {
              // Codes through `tmap`, block scales through `smap` (16-byte rows of two slots).
              int nb = 1;
              if (!merged)
                for (nb = 0; nb < T::TK / box_rows && key0 + nb * box_rows < it.k_end;) ++nb;
              const int rows = merged ? T::TK : box_rows;
              mbar_arrive_expect_tx(full_bar(stg), uint32_t(nb * rows) * 2 * (T::RB + T::SCALE_ROW));
              for (int j = 0; j < nb; ++j) {
                int phys = s_ids[rel + j];
                if (phys < 0 || phys >= a.num_blocks) {
                  report(a.status, PKV_DEV_BAD_BLOCK_ID);
                  phys = int(a.num_blocks);  // out of the tensor: the loads fill zeros
                }
                if (merged) {
                  tma_load_5d(sdst, &tmap, full_bar(stg), 0, key0 & bmask, head, c3k, phys);
                  tma_load_5d(sdst + T::KS_OFF, &smap, full_bar(stg), 0, (key0 & bmask) >> 1, head, c3k, phys);
                } else {
                  const uint32_t r0 = uint32_t(j * box_rows);
                  tma_load_5d(sdst + r0 * T::RB, &tmap, full_bar(stg), 0, 0, head, c3k, phys);
                  tma_load_5d(sdst + T::V_OFF + r0 * T::RB, &tmap, full_bar(stg), 0, 0, head, c3k + 1, phys);
                  tma_load_5d(sdst + T::KS_OFF + r0 * T::SCALE_ROW, &smap, full_bar(stg), 0, 0, head, c3k, phys);
                  tma_load_5d(sdst + T::VS_OFF + r0 * T::SCALE_ROW, &smap, full_bar(stg), 0, 0, head, c3k + 1,
                              phys);
                }
              }
            } else if (merged) {
              int phys = s_ids[rel];
              if (phys < 0 || phys >= a.num_blocks) {
                report(a.status, PKV_DEV_BAD_BLOCK_ID);
                phys = int(a.num_blocks);  // out of the tensor: the load fills zeros
              }
              mbar_arrive_expect_tx(full_bar(stg), T::HALVES * 2 * T::TK * 128);
#pragma unroll
              for (int h = 0; h < T::HALVES; ++h)
                tma_load_5d(sdst + h * T::SLAB, &tmap, full_bar(stg), h * (128 / T::ELEM), key0 & bmask, head,
                            c3k, phys);
            } else {
              int nb = 0;
              while (nb < T::TK / box_rows && key0 + nb * box_rows < it.k_end) ++nb;
              mbar_arrive_expect_tx(full_bar(stg), uint32_t(nb) * T::HALVES * 2 * box_rows * 128);
              for (int j = 0; j < nb; ++j) {
                int phys = s_ids[rel + j];
                if (phys < 0 || phys >= a.num_blocks) {
                  report(a.status, PKV_DEV_BAD_BLOCK_ID);
                  phys = int(a.num_blocks);
                }
#pragma unroll
                for (int h = 0; h < T::HALVES; ++h) {
                  const uint32_t dst = sdst + h * T::SLAB + uint32_t(j * box_rows) * 128;
                  tma_load_5d(dst, &tmap, full_bar(stg), h * (128 / T::ELEM), 0, head, c3k, phys);
                  tma_load_5d(dst + T::TK * 128, &tmap, full_bar(stg), h * (128 / T::ELEM), 0, head, c3k + 1,
                              phys);
                }
              }
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, flag, 0)) ok = false;  // also orders s_ids reuse
      }
      q = __shfl_sync(0xffffffffu, q, 0);
      if (!ok) break;
    }
    // Every item of this CTA is claimed: the kernels after this one on the stream (tcgen05
    // tiles, split merge) may be scheduled as the CTAs drain.  The tcgen05 kernel reads nothing
    // this one writes, and the merge waits for it to finish.
    pdl_trigger();
    if (!ok && lane == 0) {
      report(a.status, PKV_DEV_TIMEOUT);
      s_abort = 1;
      // Let loads already issued land before the CTA's shared memory goes away: the last tiles
      // and the query rows of the last published items.
      for (int k = 1; k <= T::NST && q - k >= 0; ++k) mbar_wait(full_bar((q - k) % T::NST), ((q - k) / T::NST) & 1, &s_wl);
      for (int k = 1; k <= T::IR && it_seq - k >= 0; ++k)
        mbar_wait(ifull_bar((it_seq - k) % T::IR), ((it_seq - k) / T::IR) & 1, &s_wl);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g4 = lane >> 2, t4 = lane & 3;
  DecOffsets<D, KV, QBF> offs;
  dec_offsets<D, KV, QBF>(offs, lane);
  int q = 0, it_seq = 0, merge_phase = 0;
  bool ok = true;
  for (;;) {
    const int slot = it_seq % T::IR;
    if (s_abort || !mbar_wait(ifull_bar(slot), (it_seq / T::IR) & 1, &s_wl)) { ok = false; break; }
    const ItemDesc d = descs[slot];
    const int R = d.n_q * a.g;
    // A decode item's slot also holds its query rows: released once they are in registers.
    const bool q_staged = d.state == 0 && R <= T::QROWS;
    __syncwarp();
    if (lane == 0 && !q_staged) mbar_arrive(iempty_bar(slot), 1);
    ++it_seq;
    if (d.state == 2) break;
    if (d.state == 1) continue;
    const int ntiles = d.ntiles;
    float c = a.softmax_scale * kLog2e;  // raw score -> log2 units
    float vscale = 1.f;
    if constexpr (KV == KV_E4M3 || KV == KV_NVFP4) {
      const int sh = d.kv_head + (h4 ? warp : 0);  // scales are per (layer, KV head): the warp's head
      c *= __ldg(a.k_scale + a.layer * a.hkv + sh);
      vscale = __ldg(a.v_scale + a.layer * a.hkv + sh);
    }
    const bool to_part = d.part_row >= 0;

    if (R <= 16) {
      // ---- decode: warps take whole tiles round-robin, S^T / O^T formulation.
      // fp8 and NVFP4 tiles dequantise to value * 2^-8 (E4M3) or * 2^-7 (E2M1 times its
      // block scale); the scores and the output scale take the power of two back, exactly.
      auto run = [&](auto nr_tag) {
        constexpr int NR = decltype(nr_tag)::value;
        DecState<D, KV, QBF, NR> st;
        const bool hw = NR == 1 && h4;  // four-head items have at most 8 rows: one row group
        const int nkt = hw ? ntiles >> 2 : ntiles;                         // key tiles of the item
        const int last_valid = d.k_end - (d.k_begin + (nkt - 1) * T::TK);  // rows of the last key tile in range
        if (hw) dec_load_q<D, KV, QBF, NR>(a, q4buf + slot * T::Q4SLOT, R, st, g4, t4, warp);
        else dec_load_q<D, KV, QBF, NR>(a, qbuf + slot * T::QSLOT, R, st, g4, t4, -1);
        __syncwarp();
        if (lane == 0) mbar_arrive(iempty_bar(slot), 1);
        int lim_min = d.k_end, lo_max = 0;
#pragma unroll
        for (int nr = 0; nr < NR; ++nr)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int r = nr * 8 + 2 * t4 + b;
            st.lim[nr][b] = (d.pos0 >= 0 && r < R) ? min(d.k_end, d.pos0 + r / a.g + 1) : d.k_end;
            st.lo[nr][b] = window_start(a.window, (d.pos0 >= 0 && r < R) ? d.pos0 + r / a.g : -1);
            lim_min = min(lim_min, st.lim[nr][b]);
            lo_max = max(lo_max, st.lo[nr][b]);
            st.m[nr][b] = -INFINITY;
            st.l[nr][b] = 0.f;
          }
        lim_min = __reduce_min_sync(0xffffffffu, lim_min);
        lo_max = __reduce_max_sync(0xffffffffu, lo_max);
#pragma unroll
        for (int nr = 0; nr < NR; ++nr)
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) st.acc[nr][mt][0] = st.acc[nr][mt][1] = st.acc[nr][mt][2] = st.acc[nr][mt][3] = 0.f;
        for (int t = warp; t < ntiles; t += 4) {
          // Owner by tile index within the item: the split of keys over warps (and so the
          // rounding of the merge) does not depend on which items this CTA ran before.
          const int qq = q + t;
          const int stg = qq % T::NST;
          if (!ok || s_abort || !mbar_wait(full_bar(stg), (qq / T::NST) & 1, &s_wl)) { ok = false; continue; }
          const uint32_t kb = stages + stg * T::STAGE_BYTES, vb = kb + T::V_OFF;
          const int kt = hw ? t >> 2 : t;  // key tile (four-head items: head kv_head + warp)
          if (kt == nkt - 1 && last_valid < T::TK) {
            if constexpr (T::FP4) zero_v_tail_fp4<T::TK, T::SCALE_ROW>(vb, kb + T::VS_OFF, last_valid, lane);
            else zero_v_tail<T::RB, T::TK, T::SLAB>(vb, last_valid, lane);
            fence_proxy_async_smem();
          }
          const int key0 = d.k_begin + kt * T::TK;
          if constexpr (T::FP4)
            dec_tile_fp4<D, QBF>(st, offs, kb, vb, kb + T::KS_OFF, kb + T::VS_OFF, key0, lane, deq_undo<KV>(c),
                                 key0 + T::TK > lim_min || key0 < lo_max);
          else
            dec_tile<D, KV, QBF, NR>(st, offs, kb, vb, kb + T::KS_OFF, kb + T::VS_OFF, key0, lane, deq_undo<KV>(c),
                                     key0 + T::TK > lim_min || key0 < lo_max);
          __syncwarp();
          if (lane == 0) mbar_arrive(empty_bar(stg), 4);
        }
        // Row sums over the eight lanes that share a row.
#pragma unroll
        for (int nr = 0; nr < NR; ++nr)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float x = st.l[nr][b];
            x += __shfl_xor_sync(0xffffffffu, x, 4);
            x += __shfl_xor_sync(0xffffffffu, x, 8);
            x += __shfl_xor_sync(0xffffffffu, x, 16);
            st.l[nr][b] = x;
          }
        if (hw) {
          // The warp's head is complete: its rows (R <= 8) go to the warp's own staging rows,
          // max and sum in the row's first two padding floats; written out below.
          float* ob = red_o + (T::IR * T::Q4SLOT + warp * T::OWARP) / 4;
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int r = 2 * t4 + (e & 1);
              if (r < R) ob[r * T::OSTRIDE + dec_dim<KV>(mt, e, g4)] = st.acc[0][mt][e];
            }
          if (g4 == 0) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              ob[(2 * t4 + b) * T::OSTRIDE + D] = st.m[0][b];
              ob[(2 * t4 + b) * T::OSTRIDE + D + 1] = st.l[0][b];
            }
          }
          return;
        }
#pragma unroll
        for (int nr = 0; nr < NR; ++nr)
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int r = nr * 8 + 2 * t4 + (e & 1);
              if (r < R) red_o[(warp * 16 + r) * D + dec_dim<KV>(mt, e, g4)] = st.acc[nr][mt][e];
            }
        if (g4 == 0) {
#pragma unroll
          for (int nr = 0; nr < NR; ++nr)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const int r = nr * 8 + 2 * t4 + b;
              red_m[warp * 16 + r] = st.m[nr][b];
              red_l[warp * 16 + r] = st.l[nr][b];
            }
        }
      };
      if constexpr (T::FP4) {
        run(std::integral_constant<int, 1>{});  // NVFP4 items carry at most 8 rows
      } else {
        if (h4 || R <= 8) run(std::integral_constant<int, 1>{});  // four-head items: at most 8 rows
        else if constexpr (!H4) run(std::integral_constant<int, 2>{});
      }
      if constexpr (H4) {
        __syncwarp();
        h4_write_rows<D, KV, QBF>(red_o + (T::IR * T::Q4SLOT + warp * T::OWARP) / 4, R, lane, a.g, a.hq,
                                  d.q_begin, d.kv_head + warp, to_part ? d.part_row + warp * R : -1,
                                  deq_undo<KV>(vscale), a.out, a.out_lse, a.part_o, a.part_lse);
        __syncwarp();  // the staging rows are rewritten by the warp's next item
        q += ntiles;
        if (!ok) break;
        continue;
      }
      mbar_arrive(merge_bar, 1);
      if (!mbar_wait(merge_bar, merge_phase, &s_wl)) ok = false;
      merge_phase ^= 1;
      // Thread t takes row r = t / TPR and DPT consecutive head dims of it (TPR threads per row,
      // rows rounded up to 4, 8 or 16, at most D / 4 threads per row so that DPT is a multiple of
      // 4: every float4 and 4-element store is aligned); it computes the row's merge factors
      // itself, so no further barrier is needed, and moves its dims as float4 reads and vector
      // stores.  D 128: DPT 4, 8, 16 for R <= 4, 8, 16; D 64: 4, 4, 8.
      {
        const int Rp = R <= 4 ? 4 : (R <= 8 ? 8 : 16);
        const int TPR = min(128 / Rp, D / 4), DPT = D / TPR;
        const int r = tid / TPR, d0 = (tid % TPR) * DPT;
        if (r < R) {
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * 16 + r]);
          float f[4], lsum = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            f[w] = M == -INFINITY ? 0.f : fast_exp2(red_m[w * 16 + r] - M);
            lsum += red_l[w * 16 + r] * f[w];
          }
          const float inv = lsum > 0.f ? deq_undo<KV>(vscale) / lsum : 0.f;
          const float lse2 = lsum > 0.f ? M + __log2f(lsum) : -INFINITY;  // log2 of the row's sum of exp2 scores
#pragma unroll
          for (int w = 0; w < 4; ++w) f[w] *= inv;
          const int64_t orow = to_part ? int64_t(d.part_row) + r
                                       : (int64_t(d.q_begin) + r / a.g) * a.hq + d.kv_head * a.g + r % a.g;
#pragma unroll 1
          for (int c = 0; c < DPT; c += 4) {
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const float4 x = *reinterpret_cast<const float4*>(red_o + (w * 16 + r) * D + d0 + c);
              o.x = fmaf(x.x, f[w], o.x);
              o.y = fmaf(x.y, f[w], o.y);
              o.z = fmaf(x.z, f[w], o.z);
              o.w = fmaf(x.w, f[w], o.w);
            }
            if (to_part) {
              *reinterpret_cast<float4*>(a.part_o + orow * D + d0 + c) = o;
            } else {
              const uint2 pk = QBF ? make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w))
                                   : make_uint2(pack_f16x2(o.x, o.y), pack_f16x2(o.z, o.w));
              *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + orow * D + d0 + c) = pk;
            }
          }
          if (tid % TPR == 0) {
            const float lse = lse2 * kLn2;
            if (to_part) a.part_lse[orow] = lse;
            else if (a.out_lse) a.out_lse[orow] = lse;
          }
        }
      }
      mbar_arrive(merge_bar, 1);
      if (!mbar_wait(merge_bar, merge_phase, &s_wl)) ok = false;
      merge_phase ^= 1;
    }
    q += ntiles;
    if (!ok) break;
  }
  if (!ok) {
    report(a.status, PKV_DEV_TIMEOUT);
    s_abort = 1;
  }
  // Second: the grid finishes only after the tcgen05 kernel beside it, so the merge that waits
  // for this grid also sees that kernel's partial states.
  if (a.pdl_role == 1 && tid == 0) pdl_wait();
}

// ---- host side -------------------------------------------------------------

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}
}  // namespace

// The pool as a 5-D tensor (innermost first): head_dim, slot, kv head, 2*layer + K|V, block.
// A box is 128 bytes of one row x box_rows slots x 1 head x box_kv (1: K or V; 2: K and V) x 1 block.
bool make_pool_map(const AttnArgs& a, int head_dim, int elem, CUtensorMapDataType dt, int box_rows, int box_kv,
                   CUtensorMap* map) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t B = uint64_t(1) << a.log2_block;
  cuuint64_t dims[5] = {cuuint64_t(head_dim), B, cuuint64_t(a.hkv), cuuint64_t(2 * a.num_layers), cuuint64_t(a.num_blocks)};
  const uint64_t row = uint64_t(head_dim) * elem;
  cuuint64_t strides[4] = {row, row * B, row * B * a.hkv, row * B * a.hkv * 2 * a.num_layers};
  cuuint32_t box[5] = {cuuint32_t(128 / elem), cuuint32_t(box_rows), 1, cuuint32_t(box_kv), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, dt, 5, const_cast<void*>(a.pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// An NVFP4 pool as two 5-D tensors over the same (block, layer, K|V, head) runs of
// B * head_dim * 9/16 bytes: the E2M1 codes (rows of head_dim/2 bytes, 64-byte swizzle) and the
// E4M3 block scales (which start B * head_dim/2 bytes into each run; viewed as 16-byte rows of
// 16 / (head_dim/16) slots, no swizzle).  Boxes: box_rows slots x 1 head x box_kv x 1 block.
bool make_fp4_maps(const AttnArgs& a, int head_dim, int box_rows, int box_kv, CUtensorMap* codes,
                   CUtensorMap* scales) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t B = uint64_t(1) << a.log2_block;
  const uint64_t rowb = uint64_t(head_dim) / 2, srow = uint64_t(head_dim) / 16;
  const uint64_t run = B * (rowb + srow);
  const uint64_t per = 16 / srow;  // slots per 16-byte scale row
  if ((B * srow) % 16 || box_rows % per) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  cuuint64_t dims[5] = {rowb, B, cuuint64_t(a.hkv), cuuint64_t(2 * a.num_layers), cuuint64_t(a.num_blocks)};
  cuuint64_t strides[4] = {rowb, run, run * a.hkv, run * a.hkv * 2 * a.num_layers};
  cuuint32_t box[5] = {cuuint32_t(rowb), cuuint32_t(box_rows), 1, cuuint32_t(box_kv), 1};
  CUresult r = fn(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(a.pool), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  void* sbase = static_cast<char*>(const_cast<void*>(a.pool)) + B * rowb;
  cuuint64_t sdims[5] = {16, B / per, cuuint64_t(a.hkv), cuuint64_t(2 * a.num_layers), cuuint64_t(a.num_blocks)};
  cuuint64_t sstrides[4] = {16, run, run * a.hkv, run * a.hkv * 2 * a.num_layers};
  cuuint32_t sbox[5] = {16, cuuint32_t(box_rows / per), 1, cuuint32_t(box_kv), 1};
  r = fn(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, sbase, sdims, sstrides, sbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The decode-tile kernel is a programmatic dependent of the plan staging: its CTAs set up their
// barriers while that runs, and wait for it before reading anything.
template <int D, int KV, bool QBF>
cudaError_t launch_tma_grid(const AttnArgs& a, int grid, cudaStream_t st, const CUtensorMap& map,
                            const CUtensorMap& smap, const TmaArgs& ta) {
  using T = TmaCfg<D, KV, QBF>;
  const cudaError_t e =
      a.heads4 ? launch_pdl(attn_tma_kernel<D, KV, QBF, true>, dim3(grid), dim3(T::THREADS), T::SMEM, st, map, smap, ta)
               : launch_pdl(attn_tma_kernel<D, KV, QBF, false>, dim3(grid), dim3(T::THREADS), T::SMEM, st, map, smap, ta);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, int KV, bool QBF>
cudaError_t launch_tma(const AttnArgs& a, int grid, cudaStream_t st) {
  using T = TmaCfg<D, KV, QBF>;
  CUtensorMap map;
  if constexpr (T::FP4) {
    const int B = 1 << a.log2_block;
    const bool merged = B >= T::TK;
    const int box_rows = merged ? T::TK : B;
    CUtensorMap smap;
    if (!make_fp4_maps(a, D, box_rows, merged ? 2 : 1, &map, &smap)) return cudaErrorInvalidValue;
    return launch_tma_grid<D, KV, QBF>(a, grid, st, map, smap, TmaArgs{a, box_rows, merged ? 1 : 0});
  }
  const CUtensorMapDataType dt = KV == KV_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : KV == KV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int B = 1 << a.log2_block;
  const bool merged = B >= T::TK;
  const int box_rows = merged ? T::TK : B;
  if (!make_pool_map(a, D, T::ELEM, dt, box_rows, merged ? 2 : 1, &map)) return cudaErrorInvalidValue;
  return launch_tma_grid<D, KV, QBF>(a, grid, st, map, map, TmaArgs{a, box_rows, merged ? 1 : 0});
}

template <int D, int KV, bool QBF>
AttnKernel tma_kernel() {
  using T = TmaCfg<D, KV, QBF>;
  // Decode-sized tiles only (larger ones are tcgen05 items).
  return AttnKernel{reinterpret_cast<const void*>(&attn_tma_kernel<D, KV, QBF, false>), T::THREADS, T::SMEM,
                    &launch_tma<D, KV, QBF>, KV == KV_NVFP4 ? PKV_FP4_ROWS : PKV_DECODE_ROWS,
                    reinterpret_cast<const void*>(&attn_tma_kernel<D, KV, QBF, true>)};
}

bool attn_tma_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k) {
  if (block_size < 8) return false;
  const bool d128 = head_dim == 128;
  if (head_dim != 64 && head_dim != 128) return false;
  switch (kv_dtype) {
    case PKV_BF16:
      if (q_dtype != PKV_BF16) return false;
      *k = d128 ? tma_kernel<128, KV_BF16, true>() : tma_kernel<64, KV_BF16, true>();
      return true;
    case PKV_F16:
      if (q_dtype != PKV_F16) return false;
      *k = d128 ? tma_kernel<128, KV_F16, false>() : tma_kernel<64, KV_F16, false>();
      return true;
    case PKV_FP8_E4M3:
      if (!d128) return false;  // 64-byte rows stay on the cp.async kernel
      if (q_dtype == PKV_BF16) *k = tma_kernel<128, KV_E4M3, true>();
      else if (q_dtype == PKV_F16) *k = tma_kernel<128, KV_E4M3, false>();
      else return false;
      return true;
    case PKV_NVFP4:
      // Decode tiles only (<= 8 rows); 16-byte block-scale rows need two slots per row and
      // 128-byte aligned scale boxes, so blocks of at least 16 slots.
      if (!d128 || block_size < 16) return false;
      if (q_dtype == PKV_BF16) *k = tma_kernel<128, KV_NVFP4, true>();
      else if (q_dtype == PKV_F16) *k = tma_kernel<128, KV_NVFP4, false>();
      else return false;
      return true;
  }
  return false;
}

}  // namespace pkv

bool pkv_heads4_capable(int kv_dtype, int head_dim, int block_size) {
  // The pools' own query dtype (fp8 and NVFP4 pools take either 16-bit query on this kernel).
  const int q_dtype = kv_dtype == PKV_F16 ? PKV_F16 : PKV_BF16;
  pkv::AttnKernel k;
  return pkv::attn_tma_kernel_for(kv_dtype, q_dtype, head_dim, block_size, &k);
}
