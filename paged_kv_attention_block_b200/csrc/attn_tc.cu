// Paged attention for tiles of more than 16 rows on bf16 / f16 pools and on fp8
// (E4M3) pools of head_dim 128: the sm_100a tensor cores (tcgen05.mma) with
// tensor-memory accumulators.
//
// Deep dive (gentlecold.top) §6 and §8: the prefill chunks of a packed batch
// are its compute-heavy part (and with prefix sharing, §10, so are the group
// tiles that put many decode rows over one shared prefix).  The work list is
// the plan's second item list; one persistent CTA per SM runs 128-row tiles,
// one tensor-memory lane and two softmax threads per row:
//
//   warp 8     TMA producer: pulls items from its atomic counter, publishes each
//              in a 4-slot descriptor ring and streams K and V tiles of 128 keys
//              into two separate rings (a K stage is released as soon as S has
//              been computed from it, a V stage once P V has), 128-byte swizzle,
//              completion counted on mbarriers.  For 16-bit pools it also loads
//              each item's Q tile, ahead of the item, into one of two Q buffers
//              (a TMA box per column slab; plain copies for listed tokens), so
//              the next item's S runs during the previous item's epilogue.  No
//              load uses cluster multicast.
//   warps 11, 12 (fp8 pools only) converters: TMA lands the one-byte codes in
//              raw rings; S reads the K codes as they are (kind::f8f6f4, with Q
//              split into a high E4M3 and a low E5M2 part), and these warps widen the V
//              codes exactly into the f16 tiles the P V MMAs read.
//   warps 9, 10 MMA issuers (one thread each): warp 10 issues S = Q K^T into one
//              of two tensor-memory S buffers, as soon as the tile's K has landed
//              and both halves of the buffer's previous P have been consumed;
//              warp 9 issues, for each half of the tile's keys, O_h += P_h V_h as
//              soon as that half's P is written.  Q (one tile per item) and K
//              come from shared memory, P from tensor memory, V from its ring as an
//              MN-major operand.  Completions are signalled with tcgen05.commit on
//              mbarriers; with two issuers one thread's commits and waits overlap
//              the other's MMAs.
//   warps 0-7  softmax, two threads per row: warps w and w + 4 share the
//              tensor-memory lanes of rows 32 (w % 4) .. + 31; warp w takes the low
//              64 keys of every tile, warp w + 4 the high 64.  Each thread keeps its
//              own running max and sum for its keys and has its own accumulator
//              (O_lo or O_hi), so the two never wait for each other inside an item:
//              per tile a thread loads its 64 scores, masks them, writes its 64
//              probabilities (16-bit) back over them and signals its half's P V.
//              Once per item the pair swaps (max, sum) through shared memory and
//              each writes half of the row's head dims from both accumulators.
//
// Tensor memory (512 columns, one CTA per SM): O_lo at 0, O_hi at D, S buffers
// at 256 and 384.  A half's P overwrites the start of that half's own S columns,
// so P is double-buffered with S and a tile's softmax never waits for the
// previous P V unless it has to rescale its accumulator.
//
// A thread's running max only moves when its tile max exceeds it by more than
// 2^8 (log2 units), so P stays <= 256 and the accumulators are rescaled rarely.
// Keys past an item's end inside its last tile are masked and their V rows
// zeroed before P V reads them.  Every wait is bounded; on a timeout the CTA
// records PKV_DEV_TIMEOUT, drains and still frees its tensor memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "attn_args.h"
#include "common.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace pkv {

// F8: fp8 (E4M3) pools, d 128.  Their tiles arrive by TMA as one-byte codes in raw rings (NRK
// stages of K, NRV of V).  S = Q K^T runs on kind::f8f6f4 straight from the raw K tiles, with Q
// split per row into a high E4M3 and a low E5M2 part after a power-of-two row scale; two converter warps widen each V tile into the f16 tile of the
// P V ring (value x 2^-8, exact).  The row scale and the K scale fold into the softmax scale, the
// power of two and the V scale into the output.
template <int D, bool F8 = false>
struct TcCfg {
  static constexpr int HALVES = D / 64;          // 64-element (128-byte) column slabs of a row
  static constexpr int TK = PKV_TC_TILE_KEYS;    // keys per tile
  static constexpr int ROWS = PKV_TILE_ROWS_TC;  // rows per item: tensor-memory lanes
  static constexpr int SLAB = TK * 128;          // one column slab of a K or V tile
  static constexpr int TILE = HALVES * SLAB;     // one K or V tile
  // stages of each ring (what the Q tile leaves of 224 KB): 2 (d 128), 6 (d 64); fp8: 2 of f16
  // tiles plus 1 of raw codes
  static constexpr int NST = F8 ? 2 : (224 * 1024 - 2 * ROWS * D * 2 - 4096) / (2 * TILE);
  static constexpr int NSK = F8 ? 0 : NST;       // f16 K stages (fp8: S reads the raw codes)
  static constexpr int RAW = F8 ? TK * D : 0;    // one fp8 K or V tile: 128 keys x D bytes
  static constexpr int NRK = F8 ? 4 : 0, NRV = F8 ? 2 : 0;  // raw K and V stages
  // the item's Q tile (K-major, 128-byte swizzle); fp8: up to three one-byte parts of it
  static constexpr int QBYTES = F8 ? 3 * ROWS * D : ROWS * D * 2;
  // 16-bit pools: two Q buffers, filled by the producer ahead of the item that uses them.
  static constexpr int NQB = F8 ? 1 : 2;
  static constexpr int IR = 4;                   // item descriptor slots
  // mbarrier indices
  // Warp roles: 0-7 softmax (two threads per row), 8 TMA producer, 9 P V issuer, 10 S issuer,
  // 11-12 fp8 converters.  Thirteen warps put four on one sub-partition, which caps registers at
  // 128 a thread (a few bytes spill); measured, two converter warps still beat one at 170.
  static constexpr int SM_WARPS = 8, SM_THREADS = 32 * SM_WARPS, PROD_WARP = 8, PV_WARP = 9, S_WARP = 10;
  static constexpr int CONV_WARP0 = 11, CONV_WARPS = F8 ? 2 : 0, CONV_THREADS = 32 * CONV_WARPS;
  static constexpr int CONSUMER_WARPS = SM_WARPS + 2 + CONV_WARPS;
  static constexpr int HALF = TK / 2;  // keys of a tile per softmax thread
  // Every POLY_EVERY-th pair of a thread's scores takes its exp2 on the FMA pipe
  // (exp2_fma2), the rest on the exp unit: the split that balances the two.
  static constexpr int POLY_EVERY = 3;
  // S, P and exchange barriers come in pairs by parity, so that a waiter is never two phases behind;
  // P and O barriers per half of the keys: PBAR + 2 h + parity, OBAR + 2 h + parity.
  static constexpr int KFULL = 0, KEMPTY = NSK, VFULL = 2 * NSK, VEMPTY = 2 * NSK + NST, IFULL = 2 * NSK + 2 * NST,
                       IEMPTY = IFULL + IR, SBAR = IEMPTY + IR, PBAR = SBAR + 2, XBAR = PBAR + 4, OBAR = XBAR + 2,
                       QBAR = OBAR + 4, QMX = QBAR + 1, QFULL = QMX + 1, QEMPTY = QFULL + 2, FIN = QEMPTY + 2, END = FIN + 1, K8FULL = END + 1,
                       K8EMPTY = K8FULL + NRK, V8FULL = K8EMPTY + NRK, V8EMPTY = V8FULL + NRV, NBAR = V8EMPTY + NRV;
  // XCHG: the two halves' (running max, sum) of every row, swapped once per item, [128 rows][2 halves].
  // QMX (fp8): the two halves' Q row maxima, [128 rows][2 halves].  fp8 Q: the high E4M3 part at
  // Q_OFF, the low E5M2 part at Q_OFF + ROWS * 128 and (f16 queries) the middle E4M3 part at
  // Q_OFF + 2 * ROWS * 128 (one 128-byte row per query row each).
  static constexpr int K_OFF = 0, V_OFF = NSK * TILE, K8_OFF = (NSK + NST) * TILE, V8_OFF = K8_OFF + NRK * RAW,
                       Q_OFF = V8_OFF + NRV * RAW, XCHG_OFF = Q_OFF + NQB * QBYTES, QMX_OFF = XCHG_OFF + ROWS * 2 * 8,
                       BAR_OFF = QMX_OFF + (F8 ? ROWS * 2 * 4 : 0),
                       DESC_OFF = BAR_OFF + (8 * NBAR + 63) / 64 * 64;
  static constexpr int SMEM = 1024 + DESC_OFF + IR * 64;
  static constexpr int THREADS = 32 * (S_WARP + 1 + CONV_WARPS);
  static constexpr int TMEM_COLS = 512;
  // Tensor-memory columns: O of the low and of the high 64 keys of every tile (D each), two S
  // buffers (fp32; each half's P at the start of its own 64 columns).
  static constexpr int O_COL = 0, S_COL = 256;
  static_assert(O_COL + 2 * D <= S_COL && S_COL + 2 * TK <= TMEM_COLS, "tensor-memory map");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(!F8 || D == 128, "fp8 tiles: head_dim 128 (128-byte rows)");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // The CTA takes all 512 tensor-memory columns: shared memory must rule out a second CTA on the SM.
  static_assert(2 * (SMEM + 1024) > 228 * 1024, "one CTA per SM");
};

struct TcDesc {
  int seq, kv_head, q_begin, n_q, k_begin, k_end, pos0, part_row, ntiles, state;  // state: 0 run, 1 skip, 2 end
  int pad[6];
};
static_assert(sizeof(TcDesc) == 64, "descriptor slot");

struct TcArgs {
  AttnArgs a;
  int32_t box_rows;  // rows per TMA box: the block size, capped at one tile
  int32_t q_tokens;  // 16-bit pools: tokens per Q box (128 / g)
};

// 3-D tiled TMA load into shared memory, completion counted on `bar` (no multicast).
PKV_DEVICE void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];\n" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Every lane waits; the warp agrees on the outcome (tcgen05.ld / st are warp-wide).
PKV_DEVICE bool warp_wait(uint32_t bar, uint32_t parity, const long long* wl) {
  const bool ok = mbar_wait(bar, parity, wl);
  return __all_sync(0xffffffffu, ok);
}

// Half hf of row r of the item (query token q_begin + r / g, or the listed token r / g of a
// shared-prefix group tile; head kv_head * g + r % g): head dims [hf * D / 2, (hf + 1) * D / 2)
// into the shared-memory Q tile, laid out as a K tile (64-dim column slabs of 128-byte rows,
// 16-byte chunk c of row r at c ^ (r & 7)).  Rows past R are zero.
template <int D>
PKV_DEVICE void tc_stage_q(const AttnArgs& a, const TcDesc& d, int R, uint32_t q_smem, int r, int hf) {
  using T = TcCfg<D>;
  const bool valid = r < R;
  const int i = valid ? r / a.g : 0;
  const int64_t token = d.pos0 <= -2 ? int64_t(__ldg(a.row_tokens + (-2 - d.pos0) + i)) : int64_t(d.q_begin) + i;
  const uint4* src = reinterpret_cast<const uint4*>(
      static_cast<const uint16_t*>(a.q) + (token * a.hq + d.kv_head * a.g + (valid ? r % a.g : 0)) * D +
      hf * (D / 2));
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
    const uint4 v = valid ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
    const int dim0 = hf * (D / 2) + 8 * j;
    const int c = (dim0 % 64) / 8;
    sts128(q_smem + uint32_t(dim0 / 64) * T::SLAB + uint32_t(r) * 128 + (uint32_t(c ^ (r & 7)) << 4), v);
  }
}

// S[128 x TK] = Q K^T (16-bit pools), one thread: D/16 MMAs of K = 16, A (Q) and B (K) both K-major in shared
// memory with the 128-byte swizzle: 8-row groups 1024 bytes apart, the k-step moving 32 bytes
// inside a 128-byte row, then to the next 64-element column slab.
template <int D, bool BF>
PKV_DEVICE void tc_mma_s(uint32_t s_tmem, uint32_t qbase, uint32_t kbase) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, T::TK, false, false);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t off = (ks >> 2) * T::SLAB + (ks & 3) * 32;
    tc::mma_ss(s_tmem, tc::smem_desc(qbase + off, 16, 1024, tc::SW128), tc::smem_desc(kbase + off, 16, 1024, tc::SW128),
               IDESC, ks > 0);
  }
}

// O[128 x D] (+)= P V over one half of a tile (64 keys), one thread: 4 MMAs of K = 16.  P comes from
// tensor memory; V is the B operand in MN-major form: 64 head dims contiguous (128 bytes, 128-byte
// swizzle), the next 64 dims one column slab further, 8 keys per 1024-byte swizzle atom, so each
// 16-key step advances 2048 bytes (vbase: the tile's first key of the half).
template <int D, bool BF>
PKV_DEVICE void tc_mma_o(uint32_t o_tmem, uint32_t p_tmem, uint32_t vbase, bool accumulate) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, D, false, true);
#pragma unroll
  for (int ks = 0; ks < T::HALF / 16; ++ks) {
    const uint64_t bd = tc::smem_desc(vbase + ks * 2048, T::SLAB, 1024, tc::SW128);
    tc::mma_ts(o_tmem, p_tmem + 8 * ks, bd, IDESC, accumulate || ks > 0);
  }
}

// S[128 x TK] = (Q_hi + Q_lo [+ Q_mid]) K^T for fp8 pools, one thread: kind::f8f6f4 MMAs of K = 32,
// A (the high E4M3, the low E5M2 and, for f16 queries, the middle E4M3 part of Q) and B (the raw K
// codes) K-major in shared memory with the 128-byte swizzle (one 128-byte row per query row / key),
// the k-step moving 32 bytes.
template <bool BF>
PKV_DEVICE void tc_mma_s_f8(uint32_t s_tmem, uint32_t qbase, uint32_t kbase) {
  constexpr uint32_t IDESC_E4 = tc::idesc_f8(128, PKV_TC_TILE_KEYS, 0), IDESC_E5 = tc::idesc_f8(128, PKV_TC_TILE_KEYS, 1);
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const uint64_t bd = tc::smem_desc(kbase + ks * 32, 16, 1024, tc::SW128);
    tc::mma_ss_f8(s_tmem, tc::smem_desc(qbase + ks * 32, 16, 1024, tc::SW128), bd, IDESC_E4, ks > 0);
    tc::mma_ss_f8(s_tmem, tc::smem_desc(qbase + 128 * 128 + ks * 32, 16, 1024, tc::SW128), bd, IDESC_E5, true);
    if constexpr (!BF)
      tc::mma_ss_f8(s_tmem, tc::smem_desc(qbase + 2 * 128 * 128 + ks * 32, 16, 1024, tc::SW128), bd, IDESC_E4, true);
  }
}

// fp8 pools: half hf of row r of the item's Q (64 of the 128 head dims, bf16 or f16) into its
// one-byte parts.  The two halves swap their maxima (barrier QMX, bounded wait) and both use the row
// scale 2^(7 - e), e = floor(log2 max|q|), which puts the row maximum in [128, 256).  bf16: high =
// E4M3(q s), low = E5M2(q s - high); f16: high = E4M3(q s), middle = E4M3(q s - high), low =
// E5M2(q s - high - middle); every rounding to nearest.  The parts sum to q s exactly: after the
// high part (4 significant bits) the residual of a bf16 q is an integer of at most 8 in units of its
// last place, which E5M2 holds; an f16 q leaves up to 64 units, of which the middle part takes all
// but at most 2.  That holds for entries down to 2^-16 of the row maximum, and the low part's
// subnormals still carry entries down to 2^-23 (an E4M3 low part stops at 2^-16: on rows spanning
// many binades that moved the log-sum-exp by 1e-2, and a two-part f16 q moved it by 2).  qs_inv = 1 / s.  Rows past
// R are zero.  Returns false when the wait runs out.
template <bool BF>
PKV_DEVICE bool tc_stage_q_f8(const AttnArgs& a, const TcDesc& d, int R, uint32_t q_smem, float* qmx, uint32_t qmx_bar,
                              int qm, int r, int hf, const long long* wl, float& qs_inv) {
  const bool valid = r < R;
  const int i = valid ? r / a.g : 0;
  const int64_t token = d.pos0 <= -2 ? int64_t(__ldg(a.row_tokens + (-2 - d.pos0) + i)) : int64_t(d.q_begin) + i;
  const uint4* src = reinterpret_cast<const uint4*>(
      static_cast<const uint16_t*>(a.q) + (token * a.hq + d.kv_head * a.g + (valid ? r % a.g : 0)) * 128 + hf * 64);
  float x[64];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 v = valid ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint16_t lo = uint16_t(w[k] & 0xffff), hi = uint16_t(w[k] >> 16);
      x[8 * j + 2 * k] = BF ? bf16_bits_to_float(lo) : __half2float(__ushort_as_half(lo));
      x[8 * j + 2 * k + 1] = BF ? bf16_bits_to_float(hi) : __half2float(__ushort_as_half(hi));
    }
  }
  float m = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j) m = fmaxf(m, fabsf(x[j]));
  qmx[r * 2 + hf] = m;
  mbar_arrive(qmx_bar, 1);
  if (!mbar_wait(qmx_bar, uint32_t(qm & 1), wl)) return false;
  m = fmaxf(m, qmx[r * 2 + (hf ^ 1)]);
  int e = m > 0.f ? int((__float_as_uint(m) >> 23) & 0xff) - 127 : 7;  // floor(log2 m) for normal m
  e = max(-119, min(e, 134));  // 2^(7 - e) and its inverse stay normal floats
  const float sc = __uint_as_float(uint32_t(127 + 7 - e) << 23);
  qs_inv = __uint_as_float(uint32_t(127 - 7 + e) << 23);
#pragma unroll
  for (int c = 0; c < 4; ++c) {  // 16-dim chunk 4 hf + c of the 128-byte row
    uint32_t hw[4], lw[4], mw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float* v = x + 16 * c + 4 * k;
      const uint32_t h01 = tc::e4m3x2_rn(v[0] * sc, v[1] * sc), h23 = tc::e4m3x2_rn(v[2] * sc, v[3] * sc);
      const float2 b01 = tc::e4m3x2_to_float2(h01), b23 = tc::e4m3x2_to_float2(h23);
      float r0 = v[0] * sc - b01.x, r1 = v[1] * sc - b01.y, r2 = v[2] * sc - b23.x, r3 = v[3] * sc - b23.y;
      if constexpr (!BF) {
        const uint32_t m01 = tc::e4m3x2_rn(r0, r1), m23 = tc::e4m3x2_rn(r2, r3);
        const float2 c01 = tc::e4m3x2_to_float2(m01), c23 = tc::e4m3x2_to_float2(m23);
        r0 -= c01.x;
        r1 -= c01.y;
        r2 -= c23.x;
        r3 -= c23.y;
        mw[k] = m01 | (m23 << 16);
      }
      hw[k] = h01 | (h23 << 16);
      lw[k] = tc::e5m2x2_rn(r0, r1) | (tc::e5m2x2_rn(r2, r3) << 16);
    }
    const uint32_t off = uint32_t(r) * 128 + (uint32_t((4 * hf + c) ^ (r & 7)) << 4);
    sts128(q_smem + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
    sts128(q_smem + 128 * 128 + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
    if constexpr (!BF) sts128(q_smem + 2 * 128 * 128 + off, make_uint4(mw[0], mw[1], mw[2], mw[3]));
  }
  return true;
}

// E4M3 codes of one 16-byte chunk -> 16 f16 values (x 2^-8), in order, as two 16-byte pieces.
PKV_DEVICE void e4m3x16_to_f16(uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t p = __byte_perm(w[i], 0, 0x3120);  // bytes (0, 2, 1, 3): pairs (0, 1) and (2, 3)
    o[2 * i] = e4m3_b02_f16x2(p);
    o[2 * i + 1] = e4m3_b13_f16x2(p);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// BF: the queries are bf16 (else f16).  F8: the pool is fp8 (MMAs then run on f16 operands).
template <int D, bool BF, bool F8>
__global__ void __launch_bounds__(TcCfg<D, F8>::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap qmap, const TcArgs ta) {
  using T = TcCfg<D, F8>;
  constexpr bool MBF = BF && !F8;  // MMA operands bf16 (else f16)
  constexpr unsigned FULL = 0xffffffffu;
  const AttnArgs& a = ta.a;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t kring = base + T::K_OFF, vring = base + T::V_OFF, k8ring = base + T::K8_OFF, v8ring = base + T::V8_OFF;
  const uint32_t bars = base + T::BAR_OFF;
  auto bar = [&](int i) { return bars + 8 * i; };
  TcDesc* descs = reinterpret_cast<TcDesc*>(base_ptr + T::DESC_OFF);
  __shared__ volatile int s_abort;
  __shared__ uint32_t s_tmem;
  __shared__ long long s_wl;  // SM cycles any one wait may take

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // This kernel may start while the decode-tile kernel ahead of it is still running: it reads
  // nothing that kernel writes (and waits for it before finishing, below).
  if (warp == 0) tc::alloc(smem_addr(&s_tmem), T::TMEM_COLS);
  if (tid == 32) {
    for (int i = 0; i < T::NSK; ++i) {
      mbar_init(bar(T::KFULL + i), 1);
      mbar_init(bar(T::KEMPTY + i), 1);
    }
    for (int i = 0; i < T::NST; ++i) {
      // F8: the f16 V tiles are filled by the converter threads, not by TMA.
      mbar_init(bar(T::VFULL + i), F8 ? T::CONV_THREADS : 1);
      mbar_init(bar(T::VEMPTY + i), 1);
    }
    for (int i = 0; i < T::NRK; ++i) {
      mbar_init(bar(T::K8FULL + i), 1);
      mbar_init(bar(T::K8EMPTY + i), 1);  // released by the S MMAs' commit
    }
    for (int i = 0; i < T::NRV; ++i) {
      mbar_init(bar(T::V8FULL + i), 1);
      mbar_init(bar(T::V8EMPTY + i), T::CONV_THREADS);
    }
    mbar_init(bar(T::QMX), T::SM_THREADS);
    for (int i = 0; i < T::IR; ++i) {
      mbar_init(bar(T::IFULL + i), 1);
      mbar_init(bar(T::IEMPTY + i), T::CONSUMER_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(T::SBAR + b), 1);
      mbar_init(bar(T::XBAR + b), T::SM_THREADS);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(T::PBAR + i), T::SM_THREADS / 2);  // the threads of one half
      mbar_init(bar(T::OBAR + i), 1);
    }
    mbar_init(bar(T::QBAR), T::SM_THREADS);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(T::QFULL + b), 1);   // the producer's arrival (with the TMA bytes, or after its copies)
      mbar_init(bar(T::QEMPTY + b), 1);  // the S issuer's commit after the item's last S
    }
    mbar_init(bar(T::FIN), 2);
    mbar_init(bar(T::END), T::CONSUMER_WARPS);
    s_abort = 0;
    s_wl = a.wait_limit;
    fence_mbar_init();
  }
  if constexpr (!F8) {
    // Rows past the last whole group of g heads are never loaded: keep them zero (finite S).
    const int rows_loaded = (T::ROWS / a.g) * a.g;
    if (tid < T::ROWS && tid >= rows_loaded)
      for (int b = 0; b < T::NQB; ++b)
        for (int h = 0; h < T::HALVES; ++h)
          for (int c = 0; c < 8; ++c) sts128(base + T::Q_OFF + b * T::QBYTES + h * T::SLAB + tid * 128 + c * 16, make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
  }
  // Second (behind the decode-tile kernel, whose CTAs had waited for the plan staging, and so
  // for the work before it, before triggering this launch): this grid reads nothing that kernel
  // writes.  First: wait for the plan staging, then let the decode-tile kernel launch beside
  // this one on the SMs it leaves free.
  if (a.pdl_role == 0) {
    pdl_wait();
    pdl_trigger();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  if (warp == T::PROD_WARP) {
    // ------------------------------------------------------------ producer
    const int total_q = __ldg(a.cu_q_lens + a.num_seqs);
    const int box_rows = ta.box_rows;
    const int lb = a.log2_block;
    const int bmask = (1 << lb) - 1;
    const int c3k = 2 * a.layer;
    int q = 0, it_seq = 0;
    bool ok = true, k_armed = false;  // k_armed: K of tile q issued, its V not yet
    int qi = 0;                       // 16-bit pools: items whose Q this warp loaded
    int next_idx = blockIdx.x;  // first item: the CTA's own index; later ones from the counter
    for (;;) {
      const int slot = it_seq % T::IR;
      int flag = 1;
      if (lane == 0) flag = mbar_wait(bar(T::IEMPTY + slot), ((it_seq / T::IR) & 1) ^ 1, &s_wl) ? 1 : 0;
      if (!__shfl_sync(FULL, flag, 0)) { ok = false; break; }
      const int idx = __shfl_sync(FULL, next_idx, 0);
      TcDesc& d = descs[slot];
      if (idx >= a.n_items) {
        if (lane == 0) {
          d.state = 2;
          mbar_arrive(bar(T::IFULL + slot), 1);
        }
        break;
      }
      if (lane == 0) next_idx = int(gridDim.x + atomicAdd(a.counter, 1u));
      const int* src = reinterpret_cast<const int*>(a.items + idx);
      const int field = lane < 8 ? __ldg(src + lane) : 0;
      PkvItem it;
      it.seq = __shfl_sync(FULL, field, 0);
      it.kv_head = __shfl_sync(FULL, field, 1);
      it.q_begin = __shfl_sync(FULL, field, 2);
      it.n_q = __shfl_sync(FULL, field, 3);
      it.k_begin = __shfl_sync(FULL, field, 4);
      it.k_end = __shfl_sync(FULL, field, 5);
      it.pos0 = __shfl_sync(FULL, field, 6);
      it.part_row = __shfl_sync(FULL, field, 7);
      const int rows = it.n_q * a.g;
      bool valid = it.seq >= 0 && it.seq < a.num_seqs && it.kv_head >= 0 && it.kv_head < a.hkv && it.n_q > 0 &&
                   rows > PKV_DECODE_ROWS && rows <= T::ROWS && it.q_begin >= 0 &&
                   (it.pos0 <= -2 || it.q_begin + it.n_q <= total_q) &&  // listed tokens: checked on the host
                   it.k_begin >= 0 && it.k_begin < it.k_end && (it.k_begin % box_rows) == 0;
      if (valid) {
        const int L = __ldg(a.seq_lens + it.seq);
        valid = it.k_end <= L && ((it.k_end - 1) >> lb) < a.max_blocks && (it.pos0 < 0 || it.pos0 + it.n_q <= L);
      }
      if (!valid && lane == 0) report(a.status, PKV_DEV_PLAN_MISMATCH);
      const int ntiles = valid ? (it.k_end - it.k_begin + T::TK - 1) / T::TK : 0;
      int qb = 0;
      if constexpr (!F8) {
        if (valid) {
          // The item's Q into buffer qi % 2, once the S MMAs of the item that used it last are
          // done: one TMA box (TOKB tokens x g heads x 64 dims) per column slab for a run of
          // tokens; plain copies for listed tokens.  Rows r = token r / g, head r % g.
          qb = qi & 1;
          int f = 1;
          if (lane == 0) f = (!s_abort && mbar_wait(bar(T::QEMPTY + qb), ((qi >> 1) & 1) ^ 1, &s_wl)) ? 1 : 0;
          if (!__shfl_sync(FULL, f, 0)) { ok = false; break; }
          const uint32_t qdst = base + T::Q_OFF + qb * T::QBYTES;
          if (it.pos0 > -2) {
            if (lane == 0) {
              mbar_arrive_expect_tx(bar(T::QFULL + qb), uint32_t(T::HALVES * 128 * a.g * ta.q_tokens));
#pragma unroll
              for (int h = 0; h < T::HALVES; ++h)
                tma_load_3d(qdst + h * T::SLAB, &qmap, bar(T::QFULL + qb), h * 64, it.kv_head * a.g, it.q_begin);
            }
          } else {
            const int R = it.n_q * a.g;
            for (int x = lane; x < R * (D / 8); x += 32) {
              const int r = x / (D / 8), ch = x % (D / 8), i = r / a.g;
              const int64_t tok = __ldg(a.row_tokens + (-2 - it.pos0) + i);
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(
                  static_cast<const uint16_t*>(a.q) + (tok * a.hq + it.kv_head * a.g + r % a.g) * D + ch * 8));
              sts128(qdst + uint32_t(ch / 8) * T::SLAB + uint32_t(r) * 128 + (uint32_t((ch % 8) ^ (r & 7)) << 4), v);
            }
            fence_proxy_async_smem();  // read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(T::QFULL + qb), 1);
          }
          ++qi;
        }
      }
      if (lane == 0) {
        d.seq = it.seq; d.kv_head = it.kv_head; d.q_begin = it.q_begin; d.n_q = it.n_q; d.k_begin = it.k_begin;
        d.k_end = it.k_end; d.pos0 = it.pos0; d.part_row = it.part_row; d.ntiles = ntiles; d.state = valid ? 0 : 1;
        d.pad[0] = qb;
        mbar_arrive(bar(T::IFULL + slot), 1);
      }
      ++it_seq;
      // Test switch: publish the item but load none of its tiles, so every consumer wait runs out.
      if (a.debug_flags & PKV_DEBUG_WITHHOLD_LOADS) continue;
      const int32_t* bt_row = a.block_tables + int64_t(it.seq) * a.max_blocks;
      for (int t = 0; t < ntiles && ok; ++t, ++q) {
        const int key0 = it.k_begin + t * T::TK;
        // One box per pool block the tile touches (one box when a block holds the whole tile);
        // lane j issues box j.
        const int nb = box_rows == T::TK ? 1 : min(T::TK / box_rows, (it.k_end - key0 + box_rows - 1) / box_rows);
        int phys = 0;
        if (lane < nb) {
          phys = __ldg(bt_row + (key0 >> lb) + lane);
          if (phys < 0 || phys >= a.num_blocks) {
            report(a.status, PKV_DEV_BAD_BLOCK_ID);
            phys = int(a.num_blocks);  // outside the tensor: the load fills zeros
          }
        }
        const int row0 = box_rows == T::TK ? (key0 & bmask) : 0;
        // The ring the TMA fills: the f16 tiles, or for fp8 pools the raw tiles.
        constexpr int NSKR = F8 ? T::NRK : T::NSK, NSVR = F8 ? T::NRV : T::NST;
        constexpr int FULL_K = F8 ? T::K8FULL : T::KFULL, EMPTY_K = F8 ? T::K8EMPTY : T::KEMPTY;
        constexpr int FULL_V = F8 ? T::V8FULL : T::VFULL, EMPTY_V = F8 ? T::V8EMPTY : T::VEMPTY;
        const uint32_t bytes = F8 ? uint32_t(nb) * box_rows * D : uint32_t(nb) * T::HALVES * box_rows * 128;
        for (int kv = 0; kv < 2; ++kv) {  // K tile, then V tile
          const int ns = kv ? NSVR : NSKR, stg = q % ns;
          const uint32_t par = ((q / ns) & 1) ^ 1;
          int f = 1;
          if (lane == 0) {
            f = (!s_abort && mbar_wait(bar((kv ? EMPTY_V : EMPTY_K) + stg), par, &s_wl)) ? 1 : 0;
            if (f) mbar_arrive_expect_tx(bar((kv ? FULL_V : FULL_K) + stg), bytes);
          }
          if (!__shfl_sync(FULL, f, 0)) { ok = false; break; }
          k_armed = kv == 0;
          if (lane < nb) {
            if constexpr (F8) {
              const uint32_t dst = (kv ? v8ring : k8ring) + stg * T::RAW + uint32_t(lane * box_rows) * D;
              tma_load_5d(dst, &tmap, bar((kv ? FULL_V : FULL_K) + stg), 0, row0, it.kv_head, c3k + kv, phys);
            } else {
              const uint32_t dst = (kv ? vring : kring) + stg * T::TILE + uint32_t(lane * box_rows) * 128;
#pragma unroll
              for (int h = 0; h < T::HALVES; ++h)
                tma_load_5d(dst + h * T::SLAB, &tmap, bar((kv ? FULL_V : FULL_K) + stg), h * 64, row0, it.kv_head,
                            c3k + kv, phys);
            }
          }
        }
      }
      if (!ok) break;
    }
    pdl_trigger();  // every item of this CTA is claimed: the split merge may be scheduled
    if (!ok && lane == 0) {
      report(a.status, PKV_DEV_TIMEOUT);
      s_abort = 1;
      // Let loads already issued land before the CTA's shared memory goes away.
      constexpr int NSKR = F8 ? T::NRK : T::NSK, NSVR = F8 ? T::NRV : T::NST;
      constexpr int FULL_K = F8 ? T::K8FULL : T::KFULL, FULL_V = F8 ? T::V8FULL : T::VFULL;
      if (k_armed) mbar_wait(bar(FULL_K + q % NSKR), (q / NSKR) & 1, &s_wl);
      for (int k = 1; k <= NSKR && q - k >= 0; ++k) mbar_wait(bar(FULL_K + (q - k) % NSKR), ((q - k) / NSKR) & 1, &s_wl);
      for (int k = 1; k <= NSVR && q - k >= 0; ++k) mbar_wait(bar(FULL_V + (q - k) % NSVR), ((q - k) / NSVR) & 1, &s_wl);
    }
    return;
  }

  if constexpr (F8) {
    if (warp >= T::CONV_WARP0) {
      // ------------------------------------------- fp8 converters (warps 11, 12)
      // V of tile qq: raw stage qq % NRV (filled by TMA) -> f16 stage qq % NST (free once the P V
      // MMAs of tile qq - NST have completed).  Chunk c (16 codes: dims 16c .. 16c+15) of
      // key row r sits at (c ^ (r & 7)) in the raw row (128-byte swizzle); its 16 f16 values go
      // to the 16-byte chunks 2(c % 4) and +1 of column slab c / 4, swizzled the same way.
      const int ct = tid - 32 * T::CONV_WARP0;
      int q = 0, it_seq = 0;
      bool ok = true;
      for (;;) {
        const int slot = it_seq % T::IR;
        bool go = __all_sync(FULL, !s_abort);
        if (go) go = warp_wait(bar(T::IFULL + slot), (it_seq / T::IR) & 1, &s_wl);
        if (!go) { ok = false; break; }
        const TcDesc d = descs[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(T::IEMPTY + slot), 1);
        ++it_seq;
        if (d.state == 2) break;
        if (d.state == 1) continue;
        for (int t = 0; t < d.ntiles && ok; ++t) {
          const int qq = q + t;
          for (int kv = 1; kv < 2 && ok; ++kv) {  // V only: S reads the raw K codes
            const int s8 = qq % T::NRV, s16 = qq % T::NST;
            go = !s_abort && warp_wait(bar((kv ? T::V8FULL : T::K8FULL) + s8), (qq / T::NRV) & 1, &s_wl);
            if (go) go = warp_wait(bar((kv ? T::VEMPTY : T::KEMPTY) + s16), ((qq / T::NST) & 1) ^ 1, &s_wl);
            if (!go) { ok = false; break; }
            const uint32_t src = (kv ? v8ring : k8ring) + s8 * T::RAW, dst = (kv ? vring : kring) + s16 * T::TILE;
            for (int x = ct; x < T::TK * 8; x += T::CONV_THREADS) {
              const int r = x >> 3, c = x & 7;
              uint4 lo, hi;
              e4m3x16_to_f16(lds128(src + uint32_t(r) * 128 + (uint32_t(c ^ (r & 7)) << 4)), lo, hi);
              const uint32_t row = dst + uint32_t(c >> 2) * T::SLAB + uint32_t(r) * 128;
              const int j = (c & 3) * 2;
              sts128(row + (uint32_t(j ^ (r & 7)) << 4), lo);
              sts128(row + (uint32_t((j + 1) ^ (r & 7)) << 4), hi);
            }
            fence_proxy_async_smem();  // the f16 tile is read by the tensor core (async proxy)
            mbar_arrive(bar((kv ? T::VFULL : T::KFULL) + s16), 1);
            mbar_arrive(bar((kv ? T::V8EMPTY : T::K8EMPTY) + s8), 1);
          }
        }
        q += d.ntiles;
        if (!ok) break;
      }
      if (!ok) {
        report(a.status, PKV_DEV_TIMEOUT);
        s_abort = 1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::END), 1);
      return;
    }
  }

  if (warp > T::PROD_WARP) {
    // ------------------------------------------- MMA issuers (9: P V, 10: S)
    // Tile qq (counted over the CTA's items) uses ring stage qq % NST, S buffer and
    // S / P / O barriers qq & 1, whose phases for that tile have parity (qq >> 1) & 1.
    const bool s_side = warp == T::S_WARP;
    int q = 0, it_seq = 0, qi_s = 0;  // qi_s: 16-bit items whose S this warp issued
    uint32_t q_ph = 0;
    bool ok = true;
    for (;;) {
      const int slot = it_seq % T::IR;
      int f = 1;
      if (lane == 0) f = (!s_abort && mbar_wait(bar(T::IFULL + slot), (it_seq / T::IR) & 1, &s_wl)) ? 1 : 0;
      if (!__shfl_sync(FULL, f, 0)) { ok = false; break; }
      const TcDesc d = descs[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::IEMPTY + slot), 1);
      ++it_seq;
      if (d.state == 2) break;
      if (d.state == 1) continue;
      const int n = d.ntiles;
      if (lane == 0) {
        bool good = true;
        if (s_side) {
          // fp8: Q staged by the softmax threads means every earlier item is finished (its
          // epilogue waited for its last P V).  16-bit: the item's Q buffer is full.
          if constexpr (F8) good = !s_abort && mbar_wait(bar(T::QBAR), q_ph, &s_wl);
          else good = !s_abort && mbar_wait(bar(T::QFULL + (qi_s & 1)), (qi_s >> 1) & 1, &s_wl);
          if (good) tc::fence_after_sync();
          for (int t = 0; t < n && good; ++t) {
            const int qq = q + t, stg = qq % T::NST;
            // The buffer's previous tile: both halves of its P (in the buffer) have been read by P V.
            // fp8: the previous item is finished (Q staged after its epilogue); 16-bit: the previous
            // item's last tiles may still be in flight, so the wait counts tiles over items.
            if (F8 ? t >= 2 : qq >= 2) {
              good = !s_abort && mbar_wait(bar(T::OBAR + (qq & 1)), ((qq - 2) >> 1) & 1, &s_wl);
              if (good) good = !s_abort && mbar_wait(bar(T::OBAR + 2 + (qq & 1)), ((qq - 2) >> 1) & 1, &s_wl);
            }
            if constexpr (F8) {
              const int s8 = qq % T::NRK;
              if (good) good = !s_abort && mbar_wait(bar(T::K8FULL + s8), (qq / T::NRK) & 1, &s_wl);
              if (!good) break;
              tc::fence_after_sync();
              tc_mma_s_f8<BF>(tmem + T::S_COL + (qq & 1) * T::TK, base + T::Q_OFF, k8ring + s8 * T::RAW);
              tc::commit(bar(T::SBAR + (qq & 1)));
              tc::commit(bar(T::K8EMPTY + s8));
            } else {
              if (good) good = !s_abort && mbar_wait(bar(T::KFULL + stg), (qq / T::NST) & 1, &s_wl);
              if (!good) break;
              tc::fence_after_sync();
              tc_mma_s<D, MBF>(tmem + T::S_COL + (qq & 1) * T::TK, base + T::Q_OFF + (qi_s & 1) * T::QBYTES,
                               kring + stg * T::TILE);
              tc::commit(bar(T::SBAR + (qq & 1)));
              tc::commit(bar(T::KEMPTY + stg));
              if (t == n - 1) tc::commit(bar(T::QEMPTY + (qi_s & 1)));  // the item's Q is no longer read
            }
          }
        } else {
          for (int t = 0; t < n && good; ++t) {
            const int qq = q + t, stg = qq % T::NST, sb = qq & 1;
            good = !s_abort && mbar_wait(bar(T::VFULL + stg), (qq / T::NST) & 1, &s_wl);
            // Each half's P V as soon as that half's P is written: O_h (+)= P_h V_h.
            for (int h = 0; h < 2 && good; ++h) {
              good = !s_abort && mbar_wait(bar(T::PBAR + 2 * h + sb), (qq >> 1) & 1, &s_wl);
              if (!good) break;
              tc::fence_after_sync();
              tc_mma_o<D, MBF>(tmem + T::O_COL + h * D, tmem + T::S_COL + sb * T::TK + h * T::HALF,
                               vring + stg * T::TILE + h * (T::HALF / 8) * 1024, t > 0);
              tc::commit(bar(T::OBAR + 2 * h + sb));
            }
            if (!good) break;
            tc::commit(bar(T::VEMPTY + stg));
          }
        }
        if (!good) {
          ok = false;
          s_abort = 1;
        }
      }
      q_ph ^= 1;
      ++qi_s;
      q += n;
      if (!__shfl_sync(FULL, ok ? 1 : 0, 0)) break;
    }
    if (lane == 0) {
      if (!ok) report(a.status, PKV_DEV_TIMEOUT);
      // Every MMA this thread issued has completed before tensor memory is released.
      tc::commit(bar(T::FIN));
      mbar_wait(bar(T::FIN), 0, &s_wl);
      tc::fence_before_sync();
      mbar_arrive(bar(T::END), 1);
    }
    return;
  }

  // ---------------------------------------------------------------- softmax
  // Split O: the thread of half hf of row r owns the keys [64 hf, 64 hf + 64) of every tile, with
  // its own running max and sum and its own accumulator O_hf, fed by the P V MMAs of those keys.
  // The two halves of a row never wait for each other during the item; its epilogue merges them.
  const int lq = warp & 3, hf = warp >> 2;  // lane quarter and key half
  const int r = 32 * lq + lane;             // row of the tile and tensor-memory lane
  const int htid = tid - hf * (T::SM_THREADS / 2);  // 0 .. 127 within the half
  const uint32_t lane_base = uint32_t(lq * 32) << 16;
  const uint32_t o_lo = tmem + lane_base + T::O_COL, o_hi = o_lo + D, o_own = o_lo + hf * D;
  const uint32_t s_tm = tmem + lane_base + T::S_COL + hf * T::HALF;  // + S buffer offset: this half's S, then its P
  float2* xchg = reinterpret_cast<float2*>(base_ptr + T::XCHG_OFF);
  int q = 0, it_seq = 0, xc = 0;  // xc: items exchanged so far (barrier XBAR + (xc & 1), parity (xc >> 1) & 1)
  int qm = 0;                     // fp8: Q row maxima swapped so far (barrier QMX, parity qm & 1)
  bool ok = true;
  for (;;) {
    const int slot = it_seq % T::IR;
    bool go = __all_sync(FULL, ok && !s_abort);
    if (go) go = warp_wait(bar(T::IFULL + slot), (it_seq / T::IR) & 1, &s_wl);
    if (!go) { ok = false; break; }
    const TcDesc d = descs[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(T::IEMPTY + slot), 1);
    ++it_seq;
    if (d.state == 2) break;
    if (d.state == 1) continue;
    const int R = d.n_q * a.g;
    const int ntiles = d.ntiles;
    float c = a.softmax_scale * kLog2e;  // raw score -> log2 units
    float vfac = 1.f;                    // output factor: the V scale of fp8 tiles
    if constexpr (F8) {
      // S comes from the raw K codes (times the row scale of Q, taken back below); the widened V
      // tiles hold code values x 2^-8, whose power of two goes back with the V scale.
      c *= __ldg(a.k_scale + a.layer * a.hkv + d.kv_head);
      vfac = __ldg(a.v_scale + a.layer * a.hkv + d.kv_head) * 256.f;
    }
    const bool to_part = d.part_row >= 0;
    const int last_valid = d.k_end - (d.k_begin + (ntiles - 1) * T::TK);  // keys of the last tile in range
    const int lim = (d.pos0 >= 0 && r < R) ? min(d.k_end, d.pos0 + r / a.g + 1) : d.k_end;
    const int lo = window_start(a.window, (d.pos0 >= 0 && r < R) ? d.pos0 + r / a.g : -1);

    // fp8: the previous item's MMAs are complete (its epilogue waited for its last P V): Q is
    // free.  16-bit pools: the producer loaded Q already.
    if constexpr (F8) {
      float qs_inv = 1.f;
      if (!tc_stage_q_f8<BF>(a, d, R, base + T::Q_OFF, reinterpret_cast<float*>(base_ptr + T::QMX_OFF), bar(T::QMX),
                             qm, r, hf, &s_wl, qs_inv)) {
        ok = false;
        break;
      }
      ++qm;
      c *= qs_inv;
    }
    if constexpr (F8) {
      fence_proxy_async_smem();  // read by the tensor core
      tc::fence_before_sync();   // the previous item's tensor-memory reads, before its next MMAs
      mbar_arrive(bar(T::QBAR), 1);
    }

    float m_run = -INFINITY, l_run = 0.f;  // running max (log2 units) and sum of this half's keys
    for (int t = 0; t < ntiles; ++t) {
      const int qq = q + t, stg = qq % T::NST, sb = qq & 1;
      go = __all_sync(FULL, ok && !s_abort);
      if (go) go = warp_wait(bar(T::SBAR + sb), (qq >> 1) & 1, &s_wl);
      if (!go) { ok = false; continue; }
      tc::fence_after_sync();
      float s[T::HALF];
      {
        uint32_t* u = reinterpret_cast<uint32_t*>(s);
#pragma unroll
        for (int c0 = 0; c0 < T::HALF; c0 += 32) tc::ld32_nowait(s_tm + sb * T::TK + c0, u + c0);
        tc::wait_ld();
        tc::keep_after_wait<T::HALF>(u);
      }
      const int key0 = d.k_begin + t * T::TK + hf * T::HALF;
      if (key0 + T::HALF > lim || key0 < lo) {
#pragma unroll
        for (int j = 0; j < T::HALF; ++j)
          if (key0 + j >= lim || key0 + j < lo) s[j] = -INFINITY;
      }
      // Max of this half over 8 independent chains.
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int j = 8; j < T::HALF; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], s[j]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float mnew = mx * c;
      float alpha = 1.f;
      bool rescale = false;
      if (mnew > m_run + 8.f) {
        alpha = fast_exp2(m_run - mnew);  // 0 while this half has seen no key
        rescale = t > 0 && m_run != -INFINITY;
        m_run = mnew;
        l_run *= alpha;
      }
      const float mneg = m_run == -INFINITY ? 0.f : -m_run;
      // p = 2^(s c - m) in pairs; partial sums over four pair chains.
      const float2 c2 = make_float2(c, c), m2 = make_float2(mneg, mneg);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int i = 0; i < T::HALF / 2; ++i) {
        const float2 x = ffma2(make_float2(s[2 * i], s[2 * i + 1]), c2, m2);
        const float2 p = (i % T::POLY_EVERY) == 0 ? exp2_fma2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
        acc[i & 3] = fadd2(acc[i & 3], p);
        s[2 * i] = p.x;
        s[2 * i + 1] = p.y;
      }
      acc[0] = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      l_run += acc[0].x + acc[0].y;
      // Keys of this half past the item's end: zero their V rows before this half's P V reads them
      // (0 * NaN would leak).
      const int zrow0 = max(last_valid, hf * T::HALF), nz = (hf + 1) * T::HALF - zrow0;
      const bool zero_tail = t == ntiles - 1 && nz > 0;
      if (zero_tail) {
        if (warp_wait(bar(T::VFULL + stg), (qq / T::NST) & 1, &s_wl)) {
          const uint32_t vt = vring + stg * T::TILE;
          for (int x = htid; x < nz * T::HALVES * 8; x += T::SM_THREADS / 2) {
            const int row = zrow0 + x / (T::HALVES * 8), h = (x / 8) % T::HALVES, ch = x % 8;
            sts128(vt + h * T::SLAB + row * 128 + (uint32_t(ch ^ (row & 7)) << 4), make_uint4(0, 0, 0, 0));
          }
        } else {
          ok = false;
        }
      }
      if (__any_sync(FULL, rescale)) {
        // O_hf must hold this half's previous P V before it is rescaled (t > 0 here).
        if (!warp_wait(bar(T::OBAR + 2 * hf + ((qq - 1) & 1)), ((qq - 1) >> 1) & 1, &s_wl)) { ok = false; continue; }
        tc::fence_after_sync();
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tc::ld32(o_own + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tc::st32(o_own + c0, o);
        }
      }
      // This half's P (16-bit pairs) at the start of its own S columns, for its P V.
      {
        uint32_t w[T::HALF / 2];
#pragma unroll
        for (int i = 0; i < T::HALF / 2; ++i)
          w[i] = MBF ? pack_bf16x2(s[2 * i], s[2 * i + 1]) : pack_f16x2(s[2 * i], s[2 * i + 1]);
        tc::st32_nowait(s_tm + sb * T::TK, w);
      }
      tc::wait_st();
      if (zero_tail) fence_proxy_async_smem();  // the zeroed V rows
      tc::fence_before_sync();
      mbar_arrive(bar(T::PBAR + 2 * hf + sb), 1);
    }
    // Epilogue: once this half's last P V is done, the halves swap (max, sum); each thread writes
    // half of the row's head dims from both accumulators:
    //   o = (O_lo 2^(m_lo - M) + O_hi 2^(m_hi - M)) / (l_lo 2^(m_lo - M) + l_hi 2^(m_hi - M)).
    go = __all_sync(FULL, ok);
    const int qlast = q + ntiles - 1;
    if (go) go = warp_wait(bar(T::OBAR + 2 * hf + (qlast & 1)), (qlast >> 1) & 1, &s_wl);
    float2 other = make_float2(-INFINITY, 0.f);
    if (go) {
      xchg[r * 2 + hf] = make_float2(m_run, l_run);
      tc::fence_before_sync();
      mbar_arrive(bar(T::XBAR + (xc & 1)), 1);
      go = warp_wait(bar(T::XBAR + (xc & 1)), (xc >> 1) & 1, &s_wl);
      other = xchg[r * 2 + (hf ^ 1)];
      ++xc;
    }
    if (go) {
      tc::fence_after_sync();
      const float M = fmaxf(m_run, other.x);
      const float f_own = m_run == -INFINITY ? 0.f : fast_exp2(m_run - M);
      const float f_oth = other.x == -INFINITY ? 0.f : fast_exp2(other.x - M);
      const float l = l_run * f_own + other.y * f_oth;
      const float inv = l > 0.f ? vfac / l : 0.f;
      const float f_lo = (hf == 0 ? f_own : f_oth) * inv, f_hi = (hf == 0 ? f_oth : f_own) * inv;
      const int64_t orow = to_part ? int64_t(d.part_row) + r
                                   : (int64_t(d.q_begin) + r / a.g) * a.hq + d.kv_head * a.g + r % a.g;
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        const int col = hf * (D / 2) + c0;
        float o[32], oh[32];
        tc::ld32(o_lo + col, o);
        tc::ld32(o_hi + col, oh);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = o[i] * f_lo + oh[i] * f_hi;
        if (r < R) {
          if (to_part) {
            float4* dst = reinterpret_cast<float4*>(a.part_o + orow * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow * D + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float* x = o + 8 * i;
              if constexpr (BF)  // the output in q's dtype
                dst[i] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                    pack_bf16x2(x[6], x[7]));
              else
                dst[i] = make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]), pack_f16x2(x[4], x[5]),
                                    pack_f16x2(x[6], x[7]));
            }
          }
        }
      }
      if (r < R && hf == 0) {
        const float lse = l > 0.f ? (M + __log2f(l)) * kLn2 : -INFINITY;
        if (to_part) a.part_lse[orow] = lse;
        else if (a.out_lse) a.out_lse[orow] = lse;
      }
    } else {
      ok = false;
    }
    q += ntiles;
    if (!ok) break;
  }
  if (!ok) {
    report(a.status, PKV_DEV_TIMEOUT);
    s_abort = 1;
  }
  // Release tensor memory once the issuers' MMAs are done and every softmax
  // warp has finished with its lanes (bounded waits; freed on every path).
  tc::fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar(T::END), 1);
  if (warp == 0) {
    if (lane == 0 && !mbar_wait(bar(T::END), 0, &s_wl)) mbar_wait(bar(T::END), 0, &s_wl);
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, T::TMEM_COLS);
    // Second: the grid finishes only after the kernel ahead of it, so the merge that waits for
    // this grid also sees that kernel's partial states.  (First: returns at once.)
    if (lane == 0) pdl_wait();
  }
}

// ---- host side -------------------------------------------------------------

namespace {
PFN_cuTensorMapEncodeTiled_v12000 q_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &res) == cudaSuccess &&
        res == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// q [total_q][Hq][D] (16-bit) as a 3-D tensor (dim, head, token); boxes of 64 dims x g heads x
// q_tokens tokens; tokens past total_q read as zeros.
bool make_q_map(const AttnArgs& a, int head_dim, CUtensorMapDataType dt, int q_tokens, CUtensorMap* map) {
  auto fn = q_encode_fn();
  if (!fn || a.total_q <= 0 || q_tokens < 1 || q_tokens > 256 || a.g > 256) return false;
  cuuint64_t dims[3] = {cuuint64_t(head_dim), cuuint64_t(a.hq), cuuint64_t(a.total_q)};
  cuuint64_t strides[2] = {cuuint64_t(head_dim) * 2, cuuint64_t(head_dim) * 2 * a.hq};
  cuuint32_t box[3] = {64, cuuint32_t(a.g), cuuint32_t(q_tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dt, 3, const_cast<void*>(a.q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}
}  // namespace

template <int D, bool BF, bool F8>
cudaError_t launch_tc(const AttnArgs& a, int grid, cudaStream_t st) {
  using T = TcCfg<D, F8>;
  CUtensorMap map;
  const int box_rows = std::min(1 << a.log2_block, T::TK);
  const CUtensorMapDataType dt = F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : (BF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (!make_pool_map(a, D, F8 ? 1 : 2, dt, box_rows, 1, &map)) return cudaErrorInvalidValue;
  // Q as (dim, head, token), boxes of 64 dims x g heads x 128 / g tokens, 128-byte swizzle: one box
  // lands a column slab of an item's Q tile in the layout the S MMAs read.
  CUtensorMap qmap{};
  const int q_tokens = T::ROWS / a.g;
  if constexpr (!F8) {
    if (!make_q_map(a, D, dt, q_tokens, &qmap)) return cudaErrorInvalidValue;
  }
  const cudaError_t e = launch_pdl(attn_tc_kernel<D, BF, F8>, dim3(grid), dim3(T::THREADS), T::SMEM, st, map, qmap,
                                   TcArgs{a, box_rows, q_tokens});
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, bool BF, bool F8 = false>
AttnKernel tc_kernel() {
  using T = TcCfg<D, F8>;
  return AttnKernel{reinterpret_cast<const void*>(&attn_tc_kernel<D, BF, F8>), T::THREADS, T::SMEM,
                    &launch_tc<D, BF, F8>, T::ROWS};
}

bool attn_tc_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k) {
  if (!pkv_tc_capable(kv_dtype, head_dim, block_size)) return false;
  const bool d128 = head_dim == 128;
  if (kv_dtype == PKV_BF16 && q_dtype == PKV_BF16) {
    *k = d128 ? tc_kernel<128, true>() : tc_kernel<64, true>();
    return true;
  }
  if (kv_dtype == PKV_F16 && q_dtype == PKV_F16) {
    *k = d128 ? tc_kernel<128, false>() : tc_kernel<64, false>();
    return true;
  }
  if (kv_dtype == PKV_FP8_E4M3 && d128 && (q_dtype == PKV_BF16 || q_dtype == PKV_F16)) {
    *k = q_dtype == PKV_BF16 ? tc_kernel<128, true, true>() : tc_kernel<128, false, true>();
    return true;
  }
  return false;
}

}  // namespace pkv

bool pkv_tc_capable(int kv_dtype, int head_dim, int block_size) {
  if (kv_dtype == PKV_FP8_E4M3) return head_dim == 128 && block_size >= 8;
  return (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16) && (head_dim == 64 || head_dim == 128) && block_size >= 8;
}

int pkv_tc_resident_ctas(int kv_dtype, int head_dim, int block_size) {
  pkv::AttnKernel k;
  const int q_dtype = kv_dtype == PKV_F16 ? PKV_F16 : PKV_BF16;
  if (!pkv::attn_tc_kernel_for(kv_dtype, q_dtype, head_dim, block_size, &k)) return -1;
  return pkv::resident_ctas(k);
}
