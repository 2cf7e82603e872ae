// Paged attention for tiles of more than 16 rows on bf16 / f16 pools: the
// sm_100a tensor cores (tcgen05.mma) with tensor-memory accumulators.
//
// Deep dive (gentlecold.top) §6 and §8: the prefill chunks of a packed batch
// are its compute-heavy part (and with prefix sharing, §10, so are the group
// tiles that put many decode rows over one shared prefix).  The work list is
// the plan's second item list; one persistent CTA per SM runs 128-row tiles,
// one tensor-memory lane and one softmax thread per row:
//
//   warp 4     TMA producer: pulls items from its atomic counter, publishes each
//              in a 4-slot descriptor ring and streams K and V tiles of 128 keys
//              into two separate rings (a K stage is released as soon as S has
//              been computed from it, a V stage once P V has), 128-byte swizzle,
//              completion counted on mbarriers.  No load uses cluster multicast.
//   warp 5     MMA issuer (one thread): S = Q K^T into one of two tensor-memory S
//              buffers, O += P V into the tensor-memory O (V read as an MN-major
//              operand straight from its ring); completions are signalled with
//              tcgen05.commit on mbarriers.  S of tile t+2 is issued as soon as
//              the softmax threads are done with S of tile t.
//   warps 0-3  softmax: stage Q once per item (K-major, 128-byte swizzle); per
//              tile load this thread's row of S, mask it, keep the row's running
//              max and sum in registers (no shuffles) and write the row of P
//              (16-bit) to shared memory; the epilogue reads the row of O from
//              tensor memory, divides by the sum and stores it.
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
  static constexpr int NST = D == 128 ? 2 : 4;   // stages of each ring
  static constexpr int QSLAB = ROWS * 128;
  static constexpr int Q_BYTES = HALVES * QSLAB;
  static constexpr int PSLAB = ROWS * 128;       // 64 keys of P
  static constexpr int P_BYTES = (TK / 64) * PSLAB;
  static constexpr int IR = 4;                   // item descriptor slots
  // mbarrier indices
  static constexpr int KFULL = 0, KEMPTY = NST, VFULL = 2 * NST, VEMPTY = 3 * NST, IFULL = 4 * NST,
                       IEMPTY = IFULL + IR, SBAR = IEMPTY + IR, PBAR = SBAR + 2, OBAR = PBAR + 1, QBAR = OBAR + 1,
                       FIN = QBAR + 1, END = FIN + 1, NBAR = END + 1;
  static constexpr int K_OFF = 0, V_OFF = NST * TILE, Q_OFF = 2 * NST * TILE, P_OFF = Q_OFF + Q_BYTES,
                       BAR_OFF = P_OFF + P_BYTES, DESC_OFF = BAR_OFF + (8 * NBAR + 63) / 64 * 64;
  static constexpr int SMEM = 1024 + DESC_OFF + IR * 64;
  static constexpr int THREADS = 192;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 128;  // S buffers at columns 128 and 256, O at column 0
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
PKV_DEVICE bool warp_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

// Row r of the item (query token q_begin + r / g, head kv_head * g + r % g) into
// the staged Q: [D / 64 column slabs][128 rows][128 B], 16-byte chunks
// XOR-swizzled by the row's low three bits (the 128-byte swizzle, K-major).
template <int D>
PKV_DEVICE void tc_stage_q(const AttnArgs& a, const TcDesc& d, int R, uint32_t qbase, int r) {
  const bool valid = r < R;
  const uint4* src = reinterpret_cast<const uint4*>(
      static_cast<const uint16_t*>(a.q) +
      ((int64_t(d.q_begin) + (valid ? r / a.g : 0)) * a.hq + d.kv_head * a.g + (valid ? r % a.g : 0)) * D);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 v = valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    sts128(qbase + uint32_t(c >> 3) * (128 * 128) + uint32_t(r) * 128 + (uint32_t((c & 7) ^ (r & 7)) << 4), v);
  }
}

// S[128 x TK] = Q K^T, one thread: D/16 MMAs of K = 16.  Q and K are K-major
// with the 128-byte swizzle: 8-row groups 1024 bytes apart, the k-step moving
// 32 bytes inside a 128-byte row, then to the next 64-element column slab.
template <int D, bool BF>
PKV_DEVICE void tc_mma_s(uint32_t s_tmem, uint32_t qbase, uint32_t kbase) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, T::TK, false, false);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint64_t ad = tc::smem_desc(qbase + (ks >> 2) * T::QSLAB + (ks & 3) * 32, 16, 1024, tc::SW128);
    const uint64_t bd = tc::smem_desc(kbase + (ks >> 2) * T::SLAB + (ks & 3) * 32, 16, 1024, tc::SW128);
    tc::mma_ss(s_tmem, ad, bd, IDESC, ks > 0);
  }
}

// O[128 x D] (+)= P V, one thread: TK/16 MMAs of K = 16.  P is K-major (two
// 64-key slabs); V is the B operand in MN-major form: 64 head dims contiguous
// (128 bytes, 128-byte swizzle), the next 64 dims one column slab further, 8
// keys per 1024-byte swizzle atom, so each 16-key step advances 2048 bytes.
template <int D, bool BF>
PKV_DEVICE void tc_mma_o(uint32_t o_tmem, uint32_t pbase, uint32_t vbase, bool accumulate) {
  using T = TcCfg<D>;
  constexpr uint32_t IDESC = tc::idesc_f16(BF, 128, D, false, true);
#pragma unroll
  for (int ks = 0; ks < T::TK / 16; ++ks) {
    const uint64_t ad = tc::smem_desc(pbase + (ks >> 2) * T::PSLAB + (ks & 3) * 32, 16, 1024, tc::SW128);
    const uint64_t bd = tc::smem_desc(vbase + ks * 2048, T::SLAB, 1024, tc::SW128);
    tc::mma_ss(o_tmem, ad, bd, IDESC, accumulate || ks > 0);
  }
}

template <int D, bool BF>
__global__ void __launch_bounds__(192, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmap, const TcArgs ta) {
  using T = TcCfg<D>;
  constexpr unsigned FULL = 0xffffffffu;
  const AttnArgs& a = ta.a;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t kring = base + T::K_OFF, vring = base + T::V_OFF, qbuf = base + T::Q_OFF, pbuf = base + T::P_OFF;
  const uint32_t bars = base + T::BAR_OFF;
  auto bar = [&](int i) { return bars + 8 * i; };
  TcDesc* descs = reinterpret_cast<TcDesc*>(base_ptr + T::DESC_OFF);
  __shared__ volatile int s_abort;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) tc::alloc(smem_addr(&s_tmem), T::TMEM_COLS);
  if (tid == 32) {
    for (int i = 0; i < T::NST; ++i) {
      mbar_init(bar(T::KFULL + i), 1);
      mbar_init(bar(T::KEMPTY + i), 1);
      mbar_init(bar(T::VFULL + i), 1);
      mbar_init(bar(T::VEMPTY + i), 1);
    }
    for (int i = 0; i < T::IR; ++i) {
      mbar_init(bar(T::IFULL + i), 1);
      mbar_init(bar(T::IEMPTY + i), 5);  // four softmax warps and the issuer
    }
    mbar_init(bar(T::SBAR), 1);
    mbar_init(bar(T::SBAR + 1), 1);
    mbar_init(bar(T::PBAR), 128);
    mbar_init(bar(T::OBAR), 1);
    mbar_init(bar(T::QBAR), 128);
    mbar_init(bar(T::FIN), 1);
    mbar_init(bar(T::END), 5);
    s_abort = 0;
    fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
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
      if (lane == 0) flag = mbar_wait(bar(T::IEMPTY + slot), ((it_seq / T::IR) & 1) ^ 1) ? 1 : 0;
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
                   rows > PKV_DECODE_ROWS && rows <= T::ROWS && it.q_begin >= 0 && it.q_begin + it.n_q <= total_q &&
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
            f = (!s_abort && mbar_wait(bar((kv ? T::VEMPTY : T::KEMPTY) + stg), par)) ? 1 : 0;
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
    if (!ok && lane == 0) {
      report(a.status, PKV_DEV_TIMEOUT);
      s_abort = 1;
      // Let loads already issued land before the CTA's shared memory goes away.
      if (k_armed) mbar_wait(bar(T::KFULL + q % T::NST), (q / T::NST) & 1);
      for (int k = 1; k <= T::NST && q - k >= 0; ++k) {
        mbar_wait(bar(T::KFULL + (q - k) % T::NST), ((q - k) / T::NST) & 1);
        mbar_wait(bar(T::VFULL + (q - k) % T::NST), ((q - k) / T::NST) & 1);
      }
    }
    return;
  }

  if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    int q = 0, it_seq = 0;
    uint32_t q_ph = 0, p_ph = 0;
    bool ok = true;
    for (;;) {
      const int slot = it_seq % T::IR;
      int f = 1;
      if (lane == 0) f = (!s_abort && mbar_wait(bar(T::IFULL + slot), (it_seq / T::IR) & 1)) ? 1 : 0;
      if (!__shfl_sync(FULL, f, 0)) { ok = false; break; }
      const TcDesc d = descs[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T::IEMPTY + slot), 1);
      ++it_seq;
      if (d.state == 2) break;
      if (d.state == 1) continue;
      const int n = d.ntiles;
      if (lane == 0) {
        auto issue_s = [&](int t) -> bool {
          const int qq = q + t, stg = qq % T::NST;
          if (s_abort || !mbar_wait(bar(T::KFULL + stg), (qq / T::NST) & 1)) return false;
          tc_mma_s<D, BF>(tmem + T::S_COL + (t & 1) * T::TK, qbuf, kring + stg * T::TILE);
          tc::commit(bar(T::SBAR + (t & 1)));
          tc::commit(bar(T::KEMPTY + stg));
          return true;
        };
        bool good = !s_abort && mbar_wait(bar(T::QBAR), q_ph);
        if (good) tc::fence_after_sync();
        for (int t = 0; t < min(2, n) && good; ++t) good = issue_s(t);
        for (int t = 0; t < n && good; ++t) {
          const int qq = q + t, stg = qq % T::NST;
          good = !s_abort && mbar_wait(bar(T::PBAR), p_ph);
          p_ph ^= 1;
          if (good) good = mbar_wait(bar(T::VFULL + stg), (qq / T::NST) & 1);
          if (!good) break;
          tc::fence_after_sync();
          tc_mma_o<D, BF>(tmem, pbuf, vring + stg * T::TILE, t > 0);
          tc::commit(bar(T::OBAR));
          tc::commit(bar(T::VEMPTY + stg));
          if (t + 2 < n) good = issue_s(t + 2);
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
      // Every MMA this CTA issued has completed before tensor memory is released.
      tc::commit(bar(T::FIN));
      mbar_wait(bar(T::FIN), 0);
      tc::fence_before_sync();
      mbar_arrive(bar(T::END), 1);
    }
    return;
  }

  // ---------------------------------------------------------------- softmax
  const int r = tid;  // row of the tile and tensor-memory lane
  const uint32_t lane_base = uint32_t(warp * 32) << 16;
  const uint32_t o_tm = tmem + lane_base, s_tm = tmem + lane_base + T::S_COL;
  int q = 0, it_seq = 0;
  uint32_t s_ph = 0, o_ph = 0;  // s_ph bit b: parity to wait for on S buffer b
  bool ok = true;
  for (;;) {
    const int slot = it_seq % T::IR;
    bool go = __all_sync(FULL, ok && !s_abort);
    if (go) go = warp_wait(bar(T::IFULL + slot), (it_seq / T::IR) & 1);
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

    // The previous item's MMAs are complete (its epilogue waited for the last P V): Q is free.
    tc_stage_q<D>(a, d, R, qbuf, r);
    fence_proxy_async_smem();
    tc::fence_before_sync();
    mbar_arrive(bar(T::QBAR), 1);

    float m_run = -INFINITY, l_run = 0.f;  // running max (log2 units) and sum of this row
    for (int t = 0; t < ntiles; ++t) {
      const int qq = q + t, stg = qq % T::NST, sb = t & 1;
      go = __all_sync(FULL, ok && !s_abort);
      if (go) go = warp_wait(bar(T::SBAR + sb), (s_ph >> sb) & 1);
      s_ph ^= 1u << sb;
      if (!go) { ok = false; continue; }
      tc::fence_after_sync();
      float s[T::TK];
#pragma unroll
      for (int c0 = 0; c0 < T::TK; c0 += 32) tc::ld32(s_tm + sb * T::TK + c0, s + c0);
      const int key0 = d.k_begin + t * T::TK;
      if (key0 + T::TK > lim) {
#pragma unroll
        for (int j = 0; j < T::TK; ++j)
          if (key0 + j >= lim) s[j] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < T::TK; ++j) mx = fmaxf(mx, s[j]);
      const float mnew = mx * c;
      float alpha = 1.f;
      bool rescale = false;
      if (mnew > m_run + 8.f) {
        alpha = fast_exp2(m_run - mnew);  // 0 while the row has seen no key
        rescale = t > 0 && m_run != -INFINITY;
        m_run = mnew;
        l_run *= alpha;
      }
      const float mneg = m_run == -INFINITY ? 0.f : -m_run;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < T::TK; ++j) {
        s[j] = fast_exp2(fmaf(s[j], c, mneg));
        rs += s[j];
      }
      l_run += rs;
      if (t == ntiles - 1 && last_valid < T::TK) {
        // Keys past the item's end: zero their V rows before P V reads them (0 * NaN would leak).
        if (warp_wait(bar(T::VFULL + stg), (qq / T::NST) & 1)) {
          const uint32_t vt = vring + stg * T::TILE;
          for (int x = tid; x < (T::TK - last_valid) * T::HALVES * 8; x += 128) {
            const int row = last_valid + x / (T::HALVES * 8), h = (x / 8) % T::HALVES, ch = x % 8;
            sts128(vt + h * T::SLAB + row * 128 + (uint32_t(ch ^ (row & 7)) << 4), make_uint4(0, 0, 0, 0));
          }
        } else {
          ok = false;
        }
      }
      if (t > 0) {  // P V of the previous tile has read P and updated O
        const bool done = warp_wait(bar(T::OBAR), o_ph);
        o_ph ^= 1;
        if (!done) { ok = false; continue; }
        tc::fence_after_sync();
      }
      if (__any_sync(FULL, rescale)) {
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tc::ld32(o_tm + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tc::st32(o_tm + c0, o);
        }
      }
#pragma unroll
      for (int ch = 0; ch < T::TK / 8; ++ch) {
        const float* x = s + 8 * ch;
        uint4 v;
        if constexpr (BF) {
          v = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                         pack_bf16x2(x[6], x[7]));
        } else {
          v = make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]), pack_f16x2(x[4], x[5]),
                         pack_f16x2(x[6], x[7]));
        }
        sts128(pbuf + (ch >> 3) * T::PSLAB + uint32_t(r) * 128 + (uint32_t((ch & 7) ^ (r & 7)) << 4), v);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(bar(T::PBAR), 1);
    }
    // Epilogue: O / l for this thread's row, straight from tensor memory.
    go = __all_sync(FULL, ok);
    if (go) go = warp_wait(bar(T::OBAR), o_ph);
    o_ph ^= 1;
    if (go) {
      tc::fence_after_sync();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const int64_t orow = to_part ? int64_t(d.part_row) + r
                                   : (int64_t(d.q_begin) + r / a.g) * a.hq + d.kv_head * a.g + r % a.g;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tc::ld32(o_tm + c0, o);
        if (r < R) {
          if (to_part) {
            float4* dst = reinterpret_cast<float4*>(a.part_o + orow * D + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow * D + c0);
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
      if (r < R) {
        const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
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
  // Release tensor memory once the issuer's MMAs are done and every softmax
  // warp has finished with its lanes (bounded waits; freed on every path).
  tc::fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar(T::END), 1);
  if (warp == 0) {
    if (lane == 0 && !mbar_wait(bar(T::END), 0)) mbar_wait(bar(T::END), 0);
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, T::TMEM_COLS);
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
  attn_tc_kernel<D, BF><<<grid, T::THREADS, T::SMEM, st>>>(map, TcArgs{a, box_rows});
  return cudaGetLastError();
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
