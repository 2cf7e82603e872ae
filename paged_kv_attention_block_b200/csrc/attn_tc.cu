// Paged attention for tiles of more than 16 rows on bf16 / f16 pools: the
// sm_100a tensor cores (tcgen05.mma) with tensor-memory accumulators.
//
// Deep dive (gentlecold.top) §6 and §8: the prefill chunks of a packed batch
// are its compute-heavy part (and with prefix sharing, §10, so are the group
// tiles that put many decode rows over one shared prefix).  The work list is
// the plan's second item list; one persistent CTA per SM runs 128-row tiles,
// one tensor-memory lane and one softmax thread per row:
//
//   warp 8     TMA producer: pulls items from its atomic counter, publishes each
//              in a 4-slot descriptor ring and streams K and V tiles of 128 keys
//              into two separate rings (a K stage is released as soon as S has
//              been computed from it, a V stage once P V has), 128-byte swizzle,
//              completion counted on mbarriers.  No load uses cluster multicast.
//   warps 9, 10 MMA issuers (one thread each): warp 10 issues S = Q K^T into one
//              of two tensor-memory S buffers, as soon as the tile's K has landed
//              and the softmax threads are done with the buffer's previous tile;
//              warp 9 issues O += P V into the tensor-memory O once a tile's P is
//              written.  Q and P are the A operands straight from tensor memory,
//              K and V the B operands from their rings (V as an MN-major operand),
//              so shared memory only carries K and V.  Completions are signalled
//              with tcgen05.commit on mbarriers; with two issuers one thread's
//              commits and waits overlap the other's MMAs.
//   warps 0-7  softmax, two threads per row: warps w and w + 4 share the
//              tensor-memory lanes of rows 32 (w % 4) .. + 31 and split every row's
//              columns in halves.  Once per item each thread writes its half of the
//              row of Q into tensor memory; per tile it loads its half of the row
//              of S, masks it, swaps its partial max with its partner through
//              shared memory, keeps the running max and its partial sum in
//              registers and writes its half of the row of P (16-bit) back to
//              tensor memory; the epilogue reads its half of the row of O, divides
//              by the row's sum and stores it.
//
// Tensor memory (512 columns, one CTA per SM): O at 0, S buffers at 128 and
// 256, Q at 384.  P of a tile overwrites the first half of its own S buffer
// (both threads of every row have loaded their S by then: the max swap sits in
// between), so P is double-buffered with S and a tile's softmax never waits for
// the previous P V unless it has to rescale O.
//
// The running max of a row only moves when the row max exceeds it by more than
// 2^8 (log2 units), so P stays <= 256 and the row of O in tensor memory is
// rescaled rarely.  Keys past an item's end inside its last tile are masked and
// their V rows zeroed before P V reads them.  Every wait is bounded; on a
// timeout the CTA records PKV_DEV_TIMEOUT, drains and still frees its tensor
// memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_args.h"
#include "common.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace pkv {

template <int D>
struct TcCfg {
  static constexpr int HALVES = D / 64;          // 64-element (128-byte) column slabs of a row
  static constexpr int TK = PKV_TC_TILE_KEYS;    // keys per tile
  static constexpr int ROWS = PKV_TILE_ROWS_TC;  // rows per item: tensor-memory lanes
  static constexpr int SLAB = TK * 128;          // one column slab of a K or V tile
  static constexpr int TILE = HALVES * SLAB;     // one K or V tile
  static constexpr int NST = (192 * 1024) / (2 * TILE);  // stages of each ring: 3 (d 128), 6 (d 64)
  static constexpr int IR = 4;                   // item descriptor slots
  // mbarrier indices
  // Warp roles: 0-7 softmax (two threads per row), 8 TMA producer, 9 P V issuer, 10 S issuer.
  static constexpr int SM_WARPS = 8, SM_THREADS = 32 * SM_WARPS, PROD_WARP = 8, PV_WARP = 9, S_WARP = 10;
  static constexpr int CONSUMER_WARPS = SM_WARPS + 2;
  static constexpr int HALF = TK / 2;  // keys of a tile per softmax thread
  // Every POLY_EVERY-th pair of a thread's scores takes its exp2 on the FMA pipe
  // (exp2_fma2), the rest on the exp unit: the split that balances the two.
  static constexpr int POLY_EVERY = 3;
  // S, P and exchange barriers come in pairs by parity, so that a waiter is never two phases behind.
  static constexpr int KFULL = 0, KEMPTY = NST, VFULL = 2 * NST, VEMPTY = 3 * NST, IFULL = 4 * NST,
                       IEMPTY = IFULL + IR, SBAR = IEMPTY + IR, PBAR = SBAR + 2, XBAR = PBAR + 2, OBAR = XBAR + 2,
                       QBAR = OBAR + 2, FIN = QBAR + 1, END = FIN + 1, NBAR = END + 1;
  // XCHG: partial row maxima / sums swapped between the two threads of a row, [2 parities][2 halves][128 rows].
  static constexpr int K_OFF = 0, V_OFF = NST * TILE, XCHG_OFF = 2 * NST * TILE, BAR_OFF = XCHG_OFF + 2 * 2 * ROWS * 4,
                       DESC_OFF = BAR_OFF + (8 * NBAR + 63) / 64 * 64;
  static constexpr int SMEM = 1024 + DESC_OFF + IR * 64;
  static constexpr int THREADS = 32 * (S_WARP + 1);
  static constexpr int TMEM_COLS = 512;
  // Tensor-memory columns: O, two S buffers (fp32; P in the first half of each), Q (16-bit pairs).
  static constexpr int O_COL = 0, S_COL = 128, Q_COL = 384;
  static_assert(Q_COL + D / 2 <= TMEM_COLS, "tensor-memory map");
  static_assert(D == 64 || D == 128, "head_dim");
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
};

// Every lane waits; the warp agrees on the outcome (tcgen05.ld / st are warp-wide).
PKV_DEVICE bool warp_wait(uint32_t bar, uint32_t parity, const long long* wl) {
  const bool ok = mbar_wait(bar, parity, wl);
  return __all_sync(0xffffffffu, ok);
}

// Half hf of row r of the item (query token q_begin + r / g, or the listed token r / g of a
// shared-prefix group tile; head kv_head * g + r % g): head dims [hf * D / 2, (hf + 1) * D / 2)
// into this thread's tensor-memory lane at q_tmem, two 16-bit values per column (the pairs are
// the row's bytes in memory order).  Rows past R are zero.
template <int D>
PKV_DEVICE void tc_stage_q(const AttnArgs& a, const TcDesc& d, int R, uint32_t q_tmem, int r, int hf) {
  const bool valid = r < R;
  const int i = valid ? r / a.g : 0;
  const int64_t token = d.pos0 <= -2 ? int64_t(__ldg(a.row_tokens + (-2 - d.pos0) + i)) : int64_t(d.q_begin) + i;
  const uint4* src = reinterpret_cast<const uint4*>(
      static_cast<const uint16_t*>(a.q) + (token * a.hq + d.kv_head * a.g + (valid ? r % a.g : 0)) * D +
      hf * (D / 2));
  uint32_t w[D / 4];
#pragma unroll
  for (int i = 0; i < D / 16; ++i) {
    const uint4 v = valid ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    w[4 * i] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
  if constexpr (D == 128) tc::st32_nowait(q_tmem, w);
  else tc::st16_nowait(q_tmem, w);
  tc::wait_st();
}

// S[128 x TK] = Q K^T, one thread: D/16 MMAs of K = 16.  Q comes from tensor
// memory (8 columns per step); K is K-major with the 128-byte swizzle: 8-row
// groups 1024 bytes apart, the k-step moving 32 bytes inside a 128-byte row,
// then to the next 64-element column slab.
template <int D, bool BF>
PKV_DEVICE void tc_mma_s(uint32_t s_tmem, uint32_t q_tmem, uint32_t kbase) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, T::TK, false, false);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint64_t bd = tc::smem_desc(kbase + (ks >> 2) * T::SLAB + (ks & 3) * 32, 16, 1024, tc::SW128);
    tc::mma_ts(s_tmem, q_tmem + 8 * ks, bd, IDESC, ks > 0);
  }
}

// O[128 x D] (+)= P V, one thread: TK/16 MMAs of K = 16.  P comes from tensor
// memory; V is the B operand in MN-major form: 64 head dims contiguous (128
// bytes, 128-byte swizzle), the next 64 dims one column slab further, 8 keys
// per 1024-byte swizzle atom, so each 16-key step advances 2048 bytes.
template <int D, bool BF>
PKV_DEVICE void tc_mma_o(uint32_t o_tmem, uint32_t p_tmem, uint32_t vbase, bool accumulate) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, D, false, true);
#pragma unroll
  for (int ks = 0; ks < T::TK / 16; ++ks) {
    const uint64_t bd = tc::smem_desc(vbase + ks * 2048, T::SLAB, 1024, tc::SW128);
    tc::mma_ts(o_tmem, p_tmem + 8 * ks, bd, IDESC, accumulate || ks > 0);
  }
}

template <int D, bool BF>
__global__ void __launch_bounds__(352, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmap, const TcArgs ta) {
  using T = TcCfg<D>;
  constexpr unsigned FULL = 0xffffffffu;
  const AttnArgs& a = ta.a;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t kring = base + T::K_OFF, vring = base + T::V_OFF;
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
  float* xchg = reinterpret_cast<float*>(base_ptr + T::XCHG_OFF);
  if (tid == 32) {
    for (int i = 0; i < T::NST; ++i) {
      mbar_init(bar(T::KFULL + i), 1);
      mbar_init(bar(T::KEMPTY + i), 1);
      mbar_init(bar(T::VFULL + i), 1);
      mbar_init(bar(T::VEMPTY + i), 1);
    }
    for (int i = 0; i < T::IR; ++i) {
      mbar_init(bar(T::IFULL + i), 1);
      mbar_init(bar(T::IEMPTY + i), T::CONSUMER_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(T::SBAR + b), 1);
      mbar_init(bar(T::PBAR + b), T::SM_THREADS);
      mbar_init(bar(T::XBAR + b), T::SM_THREADS);
      mbar_init(bar(T::OBAR + b), 1);
    }
    mbar_init(bar(T::QBAR), T::SM_THREADS);
    mbar_init(bar(T::FIN), 2);
    mbar_init(bar(T::END), T::CONSUMER_WARPS);
    s_abort = 0;
    s_wl = a.wait_limit;
    fence_mbar_init();
  }
  // Behind the decode-tile kernel, whose CTAs had waited for the plan staging (and so for the
  // work before it) before triggering this launch, this grid reads nothing that kernel writes.
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
      if (lane == 0) {
        d.seq = it.seq; d.kv_head = it.kv_head; d.q_begin = it.q_begin; d.n_q = it.n_q; d.k_begin = it.k_begin;
        d.k_end = it.k_end; d.pos0 = it.pos0; d.part_row = it.part_row; d.ntiles = ntiles; d.state = valid ? 0 : 1;
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
        const int stg = q % T::NST;
        const uint32_t par = ((q / T::NST) & 1) ^ 1;
        const uint32_t bytes = uint32_t(nb) * T::HALVES * box_rows * 128;
        for (int kv = 0; kv < 2; ++kv) {  // K tile, then V tile
          int f = 1;
          if (lane == 0) {
            f = (!s_abort && mbar_wait(bar((kv ? T::VEMPTY : T::KEMPTY) + stg), par, &s_wl)) ? 1 : 0;
            if (f) mbar_arrive_expect_tx(bar((kv ? T::VFULL : T::KFULL) + stg), bytes);
          }
          if (!__shfl_sync(FULL, f, 0)) { ok = false; break; }
          k_armed = kv == 0;
          if (lane < nb) {
            const uint32_t dst = (kv ? vring : kring) + stg * T::TILE + uint32_t(lane * box_rows) * 128;
#pragma unroll
            for (int h = 0; h < T::HALVES; ++h)
              tma_load_5d(dst + h * T::SLAB, &tmap, bar((kv ? T::VFULL : T::KFULL) + stg), h * 64, row0, it.kv_head,
                          c3k + kv, phys);
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
      if (k_armed) mbar_wait(bar(T::KFULL + q % T::NST), (q / T::NST) & 1, &s_wl);
      for (int k = 1; k <= T::NST && q - k >= 0; ++k) {
        mbar_wait(bar(T::KFULL + (q - k) % T::NST), ((q - k) / T::NST) & 1, &s_wl);
        mbar_wait(bar(T::VFULL + (q - k) % T::NST), ((q - k) / T::NST) & 1, &s_wl);
      }
    }
    return;
  }

  if (warp > T::PROD_WARP) {
    // ------------------------------------------- MMA issuers (9: P V, 10: S)
    // Tile qq (counted over the CTA's items) uses ring stage qq % NST, S buffer and
    // S / P / O barriers qq & 1, whose phases for that tile have parity (qq >> 1) & 1.
    const bool s_side = warp == T::S_WARP;
    int q = 0, it_seq = 0;
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
          // Q staged means every earlier item is finished (its epilogue waited for its last P V).
          good = !s_abort && mbar_wait(bar(T::QBAR), q_ph, &s_wl);
          if (good) tc::fence_after_sync();
          for (int t = 0; t < n && good; ++t) {
            const int qq = q + t, stg = qq % T::NST;
            // The buffer's previous tile: its P (in the buffer) has been read by P V.
            if (t >= 2) good = !s_abort && mbar_wait(bar(T::OBAR + (qq & 1)), ((qq - 2) >> 1) & 1, &s_wl);
            if (good) good = !s_abort && mbar_wait(bar(T::KFULL + stg), (qq / T::NST) & 1, &s_wl);
            if (!good) break;
            tc::fence_after_sync();
            tc_mma_s<D, BF>(tmem + T::S_COL + (qq & 1) * T::TK, tmem + T::Q_COL, kring + stg * T::TILE);
            tc::commit(bar(T::SBAR + (qq & 1)));
            tc::commit(bar(T::KEMPTY + stg));
          }
        } else {
          for (int t = 0; t < n && good; ++t) {
            const int qq = q + t, stg = qq % T::NST;
            good = !s_abort && mbar_wait(bar(T::PBAR + (qq & 1)), (qq >> 1) & 1, &s_wl);
            if (good) good = mbar_wait(bar(T::VFULL + stg), (qq / T::NST) & 1, &s_wl);
            if (!good) break;
            tc::fence_after_sync();
            tc_mma_o<D, BF>(tmem + T::O_COL, tmem + T::S_COL + (qq & 1) * T::TK, vring + stg * T::TILE, t > 0);
            tc::commit(bar(T::OBAR + (qq & 1)));
            tc::commit(bar(T::VEMPTY + stg));
          }
        }
        if (!good) {
          ok = false;
          s_abort = 1;
        }
      }
      q_ph ^= 1;
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
  const int lq = warp & 3, hf = warp >> 2;  // lane quarter and column half
  const int r = 32 * lq + lane;             // row of the tile and tensor-memory lane
  const int stid = tid;                     // 0 .. SM_THREADS - 1
  const uint32_t lane_base = uint32_t(lq * 32) << 16;
  const uint32_t o_tm = tmem + lane_base + T::O_COL + hf * (D / 2), s_tm = tmem + lane_base + T::S_COL + hf * T::HALF;
  const uint32_t q_tm = tmem + lane_base + T::Q_COL + hf * (D / 4);
  const uint32_t p_tm = tmem + lane_base + T::S_COL + hf * (T::HALF / 2);  // + S buffer offset
  int q = 0, it_seq = 0, xc = 0;  // xc: exchanges so far (barrier XBAR + (xc & 1), parity (xc >> 1) & 1)
  bool ok = true;
  // Swap a value with the row's other thread through shared memory (bounded wait).
  auto exchange = [&](float mine, float& other) -> bool {
    float* buf = xchg + (xc & 1) * 2 * T::ROWS;
    buf[hf * T::ROWS + r] = mine;
    mbar_arrive(bar(T::XBAR + (xc & 1)), 1);
    const bool done = warp_wait(bar(T::XBAR + (xc & 1)), (xc >> 1) & 1, &s_wl);
    other = buf[(hf ^ 1) * T::ROWS + r];
    ++xc;
    return done;
  };
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
    const float c = a.softmax_scale * kLog2e;  // raw score -> log2 units
    const bool to_part = d.part_row >= 0;
    const int last_valid = d.k_end - (d.k_begin + (ntiles - 1) * T::TK);  // keys of the last tile in range
    const int lim = (d.pos0 >= 0 && r < R) ? min(d.k_end, d.pos0 + r / a.g + 1) : d.k_end;
    const int lo = window_start(a.window, (d.pos0 >= 0 && r < R) ? d.pos0 + r / a.g : -1);

    // The previous item's MMAs are complete (its epilogue waited for the last P V): Q is free.
    tc_stage_q<D>(a, d, R, q_tm, r, hf);
    tc::fence_before_sync();
    mbar_arrive(bar(T::QBAR), 1);

    float m_run = -INFINITY, l_run = 0.f;  // running max of the row (log2 units), sum of this half
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
      // Max of this half over 8 independent chains, then of the row with the partner's.
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int j = 8; j < T::HALF; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], s[j]);
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      float mx_other;
      if (!exchange(mx, mx_other)) { ok = false; continue; }
      mx = fmaxf(mx, mx_other);
      const float mnew = mx * c;
      // Both threads of the row take the same decisions from the same values.
      float alpha = 1.f;
      bool rescale = false;
      if (mnew > m_run + 8.f) {
        alpha = fast_exp2(m_run - mnew);  // 0 while the row has seen no key
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
      if (t == ntiles - 1 && last_valid < T::TK) {
        // Keys past the item's end: zero their V rows before P V reads them (0 * NaN would leak).
        if (warp_wait(bar(T::VFULL + stg), (qq / T::NST) & 1, &s_wl)) {
          const uint32_t vt = vring + stg * T::TILE;
          for (int x = stid; x < (T::TK - last_valid) * T::HALVES * 8; x += T::SM_THREADS) {
            const int row = last_valid + x / (T::HALVES * 8), h = (x / 8) % T::HALVES, ch = x % 8;
            sts128(vt + h * T::SLAB + row * 128 + (uint32_t(ch ^ (row & 7)) << 4), make_uint4(0, 0, 0, 0));
          }
        } else {
          ok = false;
        }
      }
      if (__any_sync(FULL, rescale)) {
        // O must hold the previous tile's P V before it is rescaled (t > 0 here).
        if (!warp_wait(bar(T::OBAR + ((qq - 1) & 1)), ((qq - 1) >> 1) & 1, &s_wl)) { ok = false; continue; }
        tc::fence_after_sync();
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          float o[32];
          tc::ld32(o_tm + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tc::st32(o_tm + c0, o);
        }
      }
      // This half of the row of P (16-bit pairs) into tensor memory for the P V step.
      {
        uint32_t w[T::HALF / 2];
#pragma unroll
        for (int i = 0; i < T::HALF / 2; ++i)
          w[i] = BF ? pack_bf16x2(s[2 * i], s[2 * i + 1]) : pack_f16x2(s[2 * i], s[2 * i + 1]);
        tc::st32_nowait(p_tm + sb * T::TK, w);
      }
      tc::wait_st();
      if (t == ntiles - 1 && last_valid < T::TK) fence_proxy_async_smem();  // the zeroed V rows
      tc::fence_before_sync();
      mbar_arrive(bar(T::PBAR + sb), 1);
    }
    // Epilogue: this half of O / l, straight from tensor memory; l is the sum of both halves.
    go = __all_sync(FULL, ok);
    float l_other = 0.f;
    if (go) go = exchange(l_run, l_other);
    if (go) go = warp_wait(bar(T::OBAR + ((q + ntiles - 1) & 1)), ((q + ntiles - 1) >> 1) & 1, &s_wl);
    if (go) {
      tc::fence_after_sync();
      const float l = l_run + l_other;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t orow = to_part ? int64_t(d.part_row) + r
                                   : (int64_t(d.q_begin) + r / a.g) * a.hq + d.kv_head * a.g + r % a.g;
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        float o[32];
        tc::ld32(o_tm + c0, o);
        const int col = hf * (D / 2) + c0;
        if (r < R) {
          if (to_part) {
            float4* dst = reinterpret_cast<float4*>(a.part_o + orow * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow * D + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float* x = o + 8 * i;
              if constexpr (BF)
                dst[i] = make_uint4(pack_bf16x2(x[0] * inv, x[1] * inv), pack_bf16x2(x[2] * inv, x[3] * inv),
                                    pack_bf16x2(x[4] * inv, x[5] * inv), pack_bf16x2(x[6] * inv, x[7] * inv));
              else
                dst[i] = make_uint4(pack_f16x2(x[0] * inv, x[1] * inv), pack_f16x2(x[2] * inv, x[3] * inv),
                                    pack_f16x2(x[4] * inv, x[5] * inv), pack_f16x2(x[6] * inv, x[7] * inv));
            }
          }
        }
      }
      if (r < R && hf == 0) {
        const float lse = l > 0.f ? (m_run + __log2f(l)) * kLn2 : -INFINITY;
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
    // The grid finishes only after the kernel ahead of it, so the merge that waits for this
    // grid also sees that kernel's partial states.
    if (lane == 0) pdl_wait();
  }
}

// ---- host side -------------------------------------------------------------

template <int D, bool BF>
cudaError_t launch_tc(const AttnArgs& a, int grid, cudaStream_t st) {
  using T = TcCfg<D>;
  CUtensorMap map;
  const int box_rows = std::min(1 << a.log2_block, T::TK);
  if (!make_pool_map(a, D, 2, BF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, box_rows, 1,
                     &map))
    return cudaErrorInvalidValue;
  const cudaError_t e = launch_pdl(attn_tc_kernel<D, BF>, dim3(grid), dim3(T::THREADS), T::SMEM, st, map,
                                   TcArgs{a, box_rows});
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, bool BF>
AttnKernel tc_kernel() {
  using T = TcCfg<D>;
  return AttnKernel{reinterpret_cast<const void*>(&attn_tc_kernel<D, BF>), T::THREADS, T::SMEM, &launch_tc<D, BF>,
                    T::ROWS};
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
  return false;
}

}  // namespace pkv

bool pkv_tc_capable(int kv_dtype, int head_dim, int block_size) {
  return (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16) && (head_dim == 64 || head_dim == 128) && block_size >= 8;
}

int pkv_tc_resident_ctas(int kv_dtype, int head_dim, int block_size) {
  pkv::AttnKernel k;
  if (!pkv::attn_tc_kernel_for(kv_dtype, kv_dtype, head_dim, block_size, &k)) return -1;
  return pkv::resident_ctas(k);
}
