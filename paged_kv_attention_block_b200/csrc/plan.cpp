// Host-side planner: turns one in-flight batch into the work list of a
// persistent attention launch.
//
// Deep dive (gentlecold.top) §6: a batch packs context requests before
// generation requests, so one launch mixes long causal chunks with one-token
// decode rows; §8: chunks attend to the cached KV plus themselves; §10:
// sequences may share prefix blocks through radix-tree reuse.  The planner
//   1. groups consecutive sequences whose block tables start with the same
//      physical blocks (cascade): their shared keys become one dense tile per
//      group and KV head instead of one read per sequence;
//   2. cuts every (sequence, query tile) into key pieces small enough that the
//      persistent CTAs finish together, weighting a tile by its rows (compute)
//      and keys (bytes); every KV head of a tile gets the same pieces;
//   3. emits the merges that combine split ranges (and group tiles) per row.
// On 16-bit pools (and fp8 pools of head_dim 128) tiles of more than 16 rows
// (prefill chunks, shared-prefix groups) go to a second list served by the tcgen05 kernel, 128 rows a tile,
// and are split and balanced over that kernel's CTAs on their own.  Items are
// ordered heaviest first within each list; CTAs pull them from an atomic
// counter.
//
// The work is done once per (query tile, key piece) -- a "piece" below -- and
// expanded over the KV heads only when the items are written: a decode batch of
// S sequences plans S tiles, not S x Hkv.  A piece of the decode-tile list becomes
// one item per KV head, or, in a four-head plan, one item per four KV heads (each
// of the TMA-fed kernel's consumer warps then runs one head's whole key range).  Scratch vectors live per thread and
// keep their capacity across calls, so a steady-state plan allocates nothing.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <functional>
#include <iterator>
#include <vector>

#include "internal.h"
#include "plan_format.h"

namespace {

// Side-by-side estimate, measured on B200: the tensor-memory tiles' rate per CTA (16-bit and fp8
// pools, causal chunks), the decode-tile kernel's stream rate per SM (16-bit, fp8 pools) and the whole HBM stream, the
// fixed cost of a decode item per CTA, and the least gain that makes the plan run side by side.
constexpr double kTcFlopsPerSm = 4.5e12, kTcFp8FlopsPerSm = 3.6e12;
constexpr double kRegBytesPerSm = 75e9, kRegFp8BytesPerSm = 45e9, kHbmBytes = 6.0e12, kRegItemSec = 1.5e-6;
constexpr double kCorunGain = 0.95;

// One (query tile, key piece): every KV head h of it becomes an item (and, when the tile's
// keys are split or it belongs to a shared-prefix group, a merge per head).
struct Piece {
  int32_t seq, q_begin, n_q, k_begin, k_end, pos0;
  // Partial rows, -1: final output.  With h heads an item (4 for decode pieces of a four-head plan,
  // else 1), head hh's rows start at part0 + (hh / h) * part_stride + (hh % h) * n_q * g, so the
  // four heads of an item own consecutive row runs.
  int32_t part0;
  int32_t part_stride;
  uint64_t cost16;   // 16 x keys x max(1, rows / 16)
  bool tc;           // tensor-memory list
};

// A (query tile) whose keys were split or that also reads a group tile: one merge per KV head.
struct Merge {
  int32_t q_begin, n_q;
  int32_t group_part0, group_stride;  // partial row of head 0 in its group tile; -1: none
  int32_t first_piece, n_pieces;      // pieces of this tile (consecutive in the piece list)
};

struct CostRun {
  uint64_t cost16;
  uint32_t count;
};

struct Scratch {
  std::vector<Piece> pieces;
  std::vector<Merge> merges;
  std::vector<int32_t> group_of;
  std::vector<int64_t> member_part;  // per sequence: partial row of head 0 in its group tile
  std::vector<int32_t> member_stride;
  std::vector<int32_t> gmembers;     // members of every group, group after group
  std::vector<int32_t> row_tokens;   // listed query tokens of group tiles
  std::vector<int32_t> run_seqs, rest_seqs;
  std::vector<uint64_t> keys, tmp;
  std::vector<CostRun> runs;                       // tail check: runs of equal-cost items
  std::vector<uint64_t> loads_a;                   // tail check: CTA loads (a min-heap)
};

Scratch& scratch() {
  thread_local Scratch s;
  return s;
}

// Pieces ordered register-tile list first, then tensor-memory list; heaviest first within each
// list, ties in creation order.  Each piece gets the key [list bit][c_max - c, `bits` wide]
// [creation index, 20 bits] (the planner refuses 2^20 pieces or more), and a stable
// least-significant-digit radix sort over the bits above the index, in 8-bit digits, orders them:
// the indices start ascending and stability keeps ties that way.
void order_pieces(const std::vector<Piece>& ps, std::vector<uint64_t>& keys, std::vector<uint64_t>& tmp) {
  const size_t n = ps.size();
  keys.resize(n);
  tmp.resize(n);
  uint64_t c_max = 0;
  for (size_t i = 0; i < n; ++i) c_max = std::max(c_max, std::min<uint64_t>(ps[i].cost16, 0xFFFFFFFFull));
  int bits = 0;
  while (bits < 32 && (c_max >> bits) != 0) ++bits;
  for (size_t i = 0; i < n; ++i)
    keys[i] = (((uint64_t(ps[i].tc) << bits) | (c_max - std::min<uint64_t>(ps[i].cost16, 0xFFFFFFFFull))) << 20) |
              uint64_t(i);
  if (n < 2) return;
  uint32_t count[256];
  for (int shift = 20; shift < 21 + bits; shift += 8) {
    std::memset(count, 0, sizeof(count));
    for (size_t i = 0; i < n; ++i) ++count[(keys[i] >> shift) & 255];
    if (count[(keys[0] >> shift) & 255] == n) continue;  // one digit value: order unchanged
    uint32_t sum = 0;
    for (int d = 0; d < 256; ++d) { const uint32_t c = count[d]; count[d] = sum; sum += c; }
    for (size_t i = 0; i < n; ++i) tmp[count[(keys[i] >> shift) & 255]++] = keys[i];
    keys.swap(tmp);
  }
}

// 16 x the cost weight of a tile of `rows` rows: max(1, rows / 16) x 16.
inline uint64_t weight16(int rows) { return uint64_t(std::max(16, rows)); }

// m a power of two
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) & ~(m - 1); }

}  // namespace

extern "C" pkv_status pkv_attention_plan(const pkv_plan_request* req, void* plan, size_t capacity,
                                         pkv_plan_info* info) {
  if (!req || !info) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: req and info are required");
  std::memset(info, 0, sizeof(*info));
  const int S = req->num_seqs, Hq = req->num_q_heads, Hkv = req->num_kv_heads, D = req->head_dim;
  const int B = req->block_size;
  if (S < 0) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: num_seqs < 0");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)", Hq, Hkv);
  const int g = Hq / Hkv;
  if (g > PKV_TILE_ROWS) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: more than %d query heads per KV head", PKV_TILE_ROWS);
  if (D != 64 && D != 128) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: head_dim %d (64 or 128)", D);
  if (!pkv_is_pow2(B) || B < 2) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: block_size %d is not a power of two > 1", B);
  if (req->kv_dtype < PKV_F32 || req->kv_dtype > PKV_NVFP4) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: kv_dtype");
  // NVFP4 pools run on the decode kernel alone: tiles of at most 8 rows, head_dim 128, blocks of 16+ slots.
  const bool fp4 = req->kv_dtype == PKV_NVFP4;
  if (fp4 && (D != 128 || B < 16 || g > PKV_FP4_ROWS))
    return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: NVFP4 pools take head_dim 128, block_size >= 16 and at most %d "
                    "query heads per KV head", PKV_FP4_ROWS);
  if (S > 0 && (!req->cu_q_lens || !req->seq_lens)) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: null length arrays");
  if (S > 0 && req->max_blocks <= 0) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: max_blocks");
  const int window = req->window;
  if (window < 0) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: window %d < 0", window);
  if (window > 0 && !req->causal)
    return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: a limited attention window needs causal rows");
  if (req->wait_limit_kcycles < 0) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: wait_limit_kcycles < 0");
  if (req->debug_flags & ~PKV_DEBUG_WITHHOLD_LOADS)
    return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: unknown debug_flags 0x%x", req->debug_flags);
  if (req->tc_num_ctas > 0 && req->num_ctas <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: tc_num_ctas > 0 needs num_ctas > 0");
  if (req->heads_per_item != 0 && req->heads_per_item != 1 && req->heads_per_item != 4)
    return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: heads_per_item %d (0, 1 or 4)", req->heads_per_item);
  // Four-head decode items: the TMA-fed decode kernel, KV heads in fours.
  const bool h4_capable = Hkv % 4 == 0 && pkv_heads4_capable(req->kv_dtype, D, B);
  if (req->heads_per_item == 4 && !h4_capable)
    return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: four-head items need num_kv_heads a multiple of 4 and a "
                    "pool the TMA-fed decode kernel serves");
  const int32_t* cu = req->cu_q_lens;
  const int32_t* L = req->seq_lens;
  if (S > 0 && cu[0] != 0) return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: cu_q_lens[0] != 0");
  for (int s = 0; s < S; ++s) {
    const int ql = cu[s + 1] - cu[s];
    if (ql < 0 || L[s] < 0 || ql > L[s])
      return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: sequence %d has q_len %d, seq_len %d", s, ql, L[s]);
    if ((int64_t(L[s]) + B - 1) / B > req->max_blocks)
      return pkv_fail(PKV_ERR_INVALID_ARG, "attention_plan: sequence %d needs %d blocks > max_blocks %d", s,
                      (L[s] + B - 1) / B, req->max_blocks);
  }
  const bool tc = pkv_tc_capable(req->kv_dtype, D, B);
  int num_ctas = req->num_ctas;
  int tc_ctas = req->num_ctas;
  if (num_ctas <= 0) {
    pkv_status st = pkv_default_num_ctas(req->kv_dtype, D, B, &num_ctas);
    if (st != PKV_OK) return st;
    tc_ctas = tc ? pkv_tc_resident_ctas(req->kv_dtype, D, B) : num_ctas;
    if (tc_ctas <= 0) return pkv_fail(PKV_ERR_CUDA, "attention_plan: occupancy query of the tcgen05 kernel failed");
  }
  const int rows_cap = tc ? PKV_TILE_ROWS_TC : (fp4 ? PKV_FP4_ROWS : PKV_TILE_ROWS);
  const int QT = std::max(1, rows_cap / g);  // query tokens per tile
  auto is_tc = [&](int rows) { return tc && rows > PKV_DECODE_ROWS; };
  const bool causal = req->causal != 0;
  auto q_len = [&](int s) { return cu[s + 1] - cu[s]; };

  // 1. Shared-prefix groups: sequences whose tables begin with the same physical blocks (deep
  // dive §10: the radix tree hands the same prefix blocks to every request that shares it).  On
  // tensor-memory pools the sharers may lie anywhere in the batch (the batch is packed by request kind,
  // not by prefix): sequences are bucketed by their first block id and each bucket is grouped
  // greedily.  A group of consecutive sequences reads its queries as one run of tokens; any other
  // group lists its query tokens in the plan (tensor-memory tiles only).  Other pools group runs
  // of consecutive sequences.
  struct Group { int mbeg, mend, tokens; bool listed; };  // members sc.gmembers[mbeg .. mend)
  std::vector<Group> groups;
  Scratch& sc = scratch();
  sc.group_of.assign(size_t(S), -1);
  sc.gmembers.clear();
  sc.row_tokens.clear();
  // A window would cut the shared prefix differently for every member: no groups then.
  if (req->cascade && req->block_tables && S > 1 && window == 0) {
    const int32_t* bt = req->block_tables;
    const int64_t mb = req->max_blocks;
    const int min_sh = req->min_shared_tokens > 0 ? req->min_shared_tokens : 256;
    // Blocks of a sequence every query row may see in full.
    auto usable = [&](int t) { return (causal ? L[t] - q_len(t) + 1 : L[t]) / B; };
    auto candidate = [&](int t) { return q_len(t) >= 1 && q_len(t) <= QT && int64_t(usable(t)) * B >= min_sh; };
    auto common = [&](int a, int b, int lim) {
      int c = 0;
      while (c < lim && bt[a * mb + c] == bt[b * mb + c]) ++c;
      return c;
    };
    if (!tc) {
      int s = 0;
      while (s < S) {
        if (q_len(s) < 1 || q_len(s) > QT) { ++s; continue; }
        int P = usable(s), t = s + 1;
        while (t < S && q_len(t) >= 1 && q_len(t) <= QT) {
          const int c = common(s, t, std::min(P, usable(t)));
          if (int64_t(c) * B < min_sh) break;
          P = c;
          ++t;
        }
        if (t - s >= 2 && int64_t(P) * B >= min_sh) {
          const int mbeg = int(sc.gmembers.size());
          for (int m = s; m < t; ++m) sc.gmembers.push_back(m);
          groups.push_back({mbeg, int(sc.gmembers.size()), P * B, false});
          s = t;
        } else {
          ++s;
        }
      }
    } else {
      // Candidates ordered by (first block id, index); each run of one first block is grouped
      // greedily around its first member, the rest of the run trying again.
      std::vector<uint64_t>& keyed = sc.keys;
      keyed.clear();
      for (int t = 0; t < S; ++t)
        if (candidate(t)) keyed.push_back((uint64_t(uint32_t(bt[t * mb])) << 32) | uint32_t(t));
      std::sort(keyed.begin(), keyed.end());
      std::vector<int32_t>& run = sc.run_seqs;
      std::vector<int32_t>& rest = sc.rest_seqs;
      for (size_t i = 0; i < keyed.size();) {
        size_t j = i;
        run.clear();
        while (j < keyed.size() && (keyed[j] >> 32) == (keyed[i] >> 32)) run.push_back(int32_t(keyed[j++] & 0xFFFFFFFFu));
        i = j;
        while (run.size() >= 2) {
          const int s0 = run[0];
          int P = usable(s0);
          const int mbeg = int(sc.gmembers.size());
          sc.gmembers.push_back(s0);
          rest.clear();
          for (size_t k = 1; k < run.size(); ++k) {
            const int t = run[k];
            const int c = common(s0, t, std::min(P, usable(t)));
            if (int64_t(c) * B >= min_sh) {
              P = c;
              sc.gmembers.push_back(t);
            } else {
              rest.push_back(t);
            }
          }
          const int mend = int(sc.gmembers.size());
          if (mend - mbeg >= 2) {
            const bool consecutive = sc.gmembers[mend - 1] - sc.gmembers[mbeg] == mend - mbeg - 1;
            groups.push_back({mbeg, mend, P * B, !consecutive});
          } else {
            sc.gmembers.resize(size_t(mbeg));
          }
          run.swap(rest);
        }
      }
    }
    for (size_t gi = 0; gi < groups.size(); ++gi)
      for (int k = groups[gi].mbeg; k < groups[gi].mend; ++k) sc.group_of[sc.gmembers[k]] = int(gi);
  }

  std::vector<Piece>& pieces = sc.pieces;
  std::vector<Merge>& merges = sc.merges;
  pieces.clear();
  merges.clear();
  int64_t part_rows = 0;
  double total_cost[2] = {0, 0};  // register-tile list, tensor-memory list (keys x weight, all heads)
  if (!groups.empty()) {
    sc.member_part.assign(size_t(S), -1);
    sc.member_stride.assign(size_t(S), 0);
  }
  int n_groups = 0;
  // Group tiles: members packed into tiles of at most QT query tokens; the tile of head h writes
  // its partial rows at part0 + h * n * g.  A listed group keeps only tiles of more than 16 rows
  // (tensor-memory tiles); members of a smaller tile leave the group and read their prefix
  // themselves.
  for (const Group& G : groups) {
    const int32_t* gm = sc.gmembers.data();
    int a = G.mbeg;
    bool any = false;
    while (a < G.mend) {
      int b = a, n = q_len(gm[a]);
      while (b + 1 < G.mend && n + q_len(gm[b + 1]) <= QT) n += q_len(gm[++b]);
      const int rows = n * g;
      const bool t = is_tc(rows);
      if (G.listed && !t) {
        for (int m = a; m <= b; ++m) sc.group_of[gm[m]] = -1;
        a = b + 1;
        continue;
      }
      int32_t pos0 = -1;  // -2 - offset: the tile's query tokens are listed at row_tokens[offset ..]
      if (G.listed) {
        pos0 = -2 - int32_t(sc.row_tokens.size());
        for (int m = a; m <= b; ++m)
          for (int tok = cu[gm[m]]; tok < cu[gm[m] + 1]; ++tok) sc.row_tokens.push_back(tok);
      }
      int off = 0;  // the member's first token within the tile
      for (int m = a; m <= b; ++m) {
        sc.member_part[gm[m]] = part_rows + int64_t(off) * g;
        sc.member_stride[gm[m]] = rows;
        off += q_len(gm[m]);
      }
      pieces.push_back({gm[a], cu[gm[a]], n, 0, G.tokens, pos0, int32_t(part_rows), rows,
                        uint64_t(G.tokens) * weight16(rows), t});
      part_rows += int64_t(rows) * Hkv;
      total_cost[t] += double(G.tokens) * double(weight16(rows)) / 16.0 * Hkv;
      any = true;
      a = b + 1;
    }
    n_groups += any ? 1 : 0;
  }
  const size_t n_group_pieces = pieces.size();

  // 2. Query tiles: (sequence, first token, tokens, keys [k0, ke), first position).
  struct Tile { int32_t seq, q_begin, n_q, k0, ke, pos0; };
  std::vector<Tile> tiles;
  tiles.reserve(size_t(S));
  for (int s = 0; s < S; ++s) {
    const int ql = q_len(s);
    if (ql == 0) continue;
    const int kb = sc.group_of[s] >= 0 ? groups[sc.group_of[s]].tokens : 0;
    for (int i0 = 0; i0 < ql; i0 += QT) {
      const int n = std::min(QT, ql - i0);
      const int ke = causal ? L[s] - ql + i0 + n : L[s];
      const int pos0 = causal ? L[s] - ql + i0 : -1;
      // Under a window the tile's first row sees keys from pos0 - window + 1 on; the range starts
      // there, rounded down to 128 keys (the kernels' tile alignment), and rows mask the rest.
      const int k0 = window > 0 ? std::max(kb, int(std::max(0, pos0 - window + 1) / 128 * 128)) : kb;
      tiles.push_back({s, cu[s] + i0, n, k0, ke, pos0});
      total_cost[is_tc(n * g)] += double(std::max(0, ke - k0)) * double(weight16(n * g)) / 16.0 * Hkv;
    }
  }

  // 2a. KV heads per decode-tile item.  A one-head item's keys are split over the kernel's four
  // consumer warps, whose states merge at the item's end, and each item costs its CTA a fixed
  // setup; items of four heads give each warp one head for the whole range, with no merge and a
  // quarter of the items.  Automatic choice: four heads on NVFP4 pools (instruction-bound tiles,
  // where the warps' merge and its barrier cost more than the extra partial rows of shorter
  // pieces) and, on the others, when the decode tiles' key ranges average at most half the
  // per-CTA share of the decode list (short ranges, where the fixed cost per item counts); long
  // ranges keep one head an item, which splits them less.
  int hpi = 1;
  {
    bool fits = h4_capable;  // every decode-sized tile of at most PKV_HEADS4_ROWS rows
    int64_t dec_tiles = 0;
    double dec_keys = 0;
    for (size_t i = 0; i < n_group_pieces; ++i)
      if (!pieces[i].tc) {
        fits = fits && pieces[i].n_q * g <= PKV_HEADS4_ROWS;
        ++dec_tiles;
        dec_keys += double(pieces[i].k_end - pieces[i].k_begin);
      }
    for (const Tile& t : tiles)
      if (!is_tc(t.n_q * g)) {
        fits = fits && t.n_q * g <= PKV_HEADS4_ROWS;
        ++dec_tiles;
        dec_keys += double(std::max(0, t.ke - t.k0));
      }
    if (req->heads_per_item == 4) {
      if (!fits)
        return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: four-head items take decode tiles of at most %d rows",
                        PKV_HEADS4_ROWS);
      hpi = dec_tiles > 0 ? 4 : 1;
    } else if (req->heads_per_item == 0 && fits && dec_tiles > 0) {
      const double share = total_cost[0] / (double(num_ctas) * 2.0);  // keys x heads per item, one head
      if (fp4 || 2.0 * dec_keys / double(dec_tiles) <= share) hpi = 4;
    }
    if (hpi == 4)
      for (size_t i = 0; i < n_group_pieces; ++i)
        if (!pieces[i].tc) pieces[i].part_stride *= 4;  // part0 + hh * rows for every head hh
  }
  auto heads_of = [&](bool t) { return t ? 1 : hpi; };  // KV heads per item of a list

  // 2b. Side by side.  With both decode-sized tiles (HBM-bound) and tensor-memory tiles
  // (tensor-bound) in the batch, the tcgen05 kernel may take k SMs and the decode-tile kernel the
  // others at the same time instead of one after the other.  Estimated times: the tensor-memory
  // list at kTcFlopsPerSm a CTA (in whole rounds of its unsplit group tiles), the decode-tile list
  // at the smaller of the HBM stream rate and kRegBytesPerSm an SM, plus kRegItemSec per item and
  // CTA.  Only for automatic CTA counts.
  bool corun = false;
  if (req->tc_num_ctas > 0) {
    if (tc && total_cost[0] > 0 && total_cost[1] > 0) {
      corun = true;
      tc_ctas = req->tc_num_ctas;
    }
  } else if (req->tc_num_ctas == 0 && req->num_ctas <= 0 && tc && total_cost[0] > 0 && total_cost[1] > 0) {
    const int sms = tc_ctas;  // one tcgen05 CTA an SM
    const int per_sm = std::max(1, num_ctas / std::max(1, sms));
    const bool f8 = req->kv_dtype == PKV_FP8_E4M3;
    const double flops = total_cost[1] * 16.0 * 4.0 * D;           // rows x keys x 4 head_dim
    const double bytes = total_cost[0] * 2.0 * D * (f8 ? 1.0 : 2.0);  // K and V rows of every key
    int64_t n_reg_pieces = 0;  // decode-tile items before any key split
    for (size_t i = 0; i < n_group_pieces; ++i) n_reg_pieces += pieces[i].tc ? 0 : 1;
    for (const Tile& t : tiles) n_reg_pieces += is_tc(t.n_q * g) ? 0 : 1;
    const double reg_items = double(n_reg_pieces) * Hkv / hpi;
    const double tc_rate = f8 ? kTcFp8FlopsPerSm : kTcFlopsPerSm;
    // Shared-prefix group tiles are never split: k CTAs take them in ceil(G / k) rounds of the
    // largest one at least (128 tiles: 64 CTAs finish in two rounds, 63 need three).
    double g_items = 0, g_flops = 0;
    for (size_t i = 0; i < n_group_pieces; ++i)
      if (pieces[i].tc) {
        g_items += Hkv;
        g_flops = std::max(g_flops, double(pieces[i].cost16) * 4.0 * D);
      }
    auto t_tc = [&](int k) {
      return std::max(flops / double(k), std::ceil(g_items / double(k)) * g_flops) / tc_rate;
    };
    auto t_reg = [&](int n) {
      return bytes / std::min(kHbmBytes, double(n) * (f8 ? kRegFp8BytesPerSm : kRegBytesPerSm)) +
             reg_items * kRegItemSec / double(n * per_sm);
    };
    const double serial = t_tc(sms) + t_reg(sms);
    double best = serial;
    int best_k = 0;
    for (int k = 1; k < sms; ++k) {
      const double t = std::max(t_tc(k), t_reg(sms - k));
      if (t < best) { best = t; best_k = k; }
    }
    if (best_k > 0 && best < kCorunGain * serial) {
      corun = true;
      tc_ctas = best_k;
      num_ctas = (sms - best_k) * per_sm;
    }
  }

  // 3. Key-range split and merges.
  const double target[2] = {total_cost[0] / (double(num_ctas) * 2.0), total_cost[1] / (double(tc_ctas) * 3.0)};
  // Longest key range of one item of a tile's list; the automatic length (about two items per
  // CTA on the decode kernel, three on the tcgen05 kernel, whose CTAs take items in turn
  // from a longer queue and whose merges spread over 16-row chunks; a four-head item a quarter
  // of a one-head item's keys, but at least 512, so that short ranges such as shared-prefix
  // members' suffixes stay whole and merge two parts) is scaled by `mult`.
  auto max_keys_for = [&](int rows, bool t, double mult) -> int32_t {
    const int64_t tile_keys = t ? PKV_TC_TILE_KEYS : PKV_TILE_KEYS;
    int64_t max_keys;
    if (req->kv_split < 0) max_keys = INT32_MAX;
    else if (req->kv_split > 0) max_keys = round_up(req->kv_split, tile_keys);
    else max_keys = std::max<int64_t>(std::max<int64_t>(heads_of(t) == 4 ? 512 : 256, 2 * tile_keys),
                                      round_up(int64_t(std::ceil(target[t] * mult * 16.0 /
                                                                 (double(weight16(rows)) * heads_of(t)))),
                                               tile_keys));
    return int32_t(std::min<int64_t>(max_keys, INT32_MAX / 2));
  };
  // Pieces of a range of n keys split into pieces of at most mk keys: nseg pieces of `seg` keys
  // (a multiple of the tile), the last one shorter.
  auto split = [](int n, int32_t mk, int64_t tile_keys, int32_t& nseg, int64_t& seg) {
    nseg = n == 0 ? 0 : int32_t((uint32_t(n) + uint32_t(mk) - 1u) / uint32_t(mk));
    seg = nseg == 0 ? 0 : round_up(int64_t((uint32_t(n) + uint32_t(nseg) - 1u) / uint32_t(nseg)), tile_keys);
  };
  // Tail check of the register-tile list.  The CTAs take items heaviest first from a counter, so
  // when the item count only just passes a multiple of the CTA count (a batch of equal long
  // ranges split into equal pieces), a few CTAs run one extra round while the rest idle.  Then
  // longer pieces are tried, and the one with the shortest simulated schedule (the greedy
  // assignment the counter produces, constant per-CTA speed) is kept if it is 2 % shorter.
  double reg_mult = 1.0;
  if (req->kv_split == 0) {
    auto count_items = [&](double mult) {
      size_t n_items = 0;
      for (size_t i = 0; i < n_group_pieces; ++i) n_items += pieces[i].tc ? 0 : size_t(Hkv / hpi);
      int last = -1;
      int32_t m = 0;
      for (const Tile& t : tiles) {
        const int rows = t.n_q * g;
        if (is_tc(rows)) continue;
        if (rows != last) { m = max_keys_for(rows, false, mult); last = rows; }
        int32_t nseg;
        int64_t seg;
        split(std::max(0, t.ke - t.k0), m, PKV_TILE_KEYS, nseg, seg);
        n_items += size_t(nseg) * size_t(Hkv / hpi);
      }
      return n_items;
    };
    const size_t N = count_items(1.0), C = size_t(num_ctas);
    // A longer piece length that leaves the item count unchanged leaves every tile's piece count,
    // and so the plan, unchanged (piece counts only fall as the length grows): nothing to try
    // when even the longest candidate gives N items (shared-prefix suffixes, already whole).
    if (N > C && N < 4 * C && (N % C) * 4 < C && count_items(1.5) != N) {
      // The counter's greedy assignment, simulated: items come heaviest first and each goes to
      // the least loaded CTA (a min-heap of the CTAs' loads; which of equally loaded CTAs takes
      // an item does not change the loads).  This branch has fewer than 4 items a CTA, so a
      // simulation is O(items log CTAs) whatever the number of distinct item costs.
      std::vector<CostRun>& runs = sc.runs;
      std::vector<uint64_t>& A = sc.loads_a;
      auto makespan = [&](double mult) {
        runs.clear();
        for (size_t i = 0; i < n_group_pieces; ++i)  // shared-prefix group items, never split
          if (!pieces[i].tc) runs.push_back({pieces[i].cost16 * uint64_t(hpi), uint32_t(Hkv / hpi)});
        int last = -1;
        int32_t m = 0;
        for (const Tile& t : tiles) {
          const int rows = t.n_q * g;
          if (is_tc(rows)) continue;
          if (rows != last) { m = max_keys_for(rows, false, mult); last = rows; }
          const int n = std::max(0, t.ke - t.k0);
          int32_t nseg;
          int64_t seg;
          split(n, m, PKV_TILE_KEYS, nseg, seg);
          if (nseg == 0) continue;
          const uint64_t w16 = weight16(rows) * uint64_t(hpi);
          if (nseg > 1) runs.push_back({uint64_t(seg) * w16, uint32_t(nseg - 1) * uint32_t(Hkv / hpi)});
          runs.push_back({uint64_t(n - (nseg - 1) * seg) * w16, uint32_t(Hkv / hpi)});
        }
        std::sort(runs.begin(), runs.end(), [](const CostRun& x, const CostRun& y) { return x.cost16 > y.cost16; });
        A.assign(size_t(num_ctas), 0);  // all zero: already a heap
        const auto later = std::greater<uint64_t>();
        for (const CostRun& run : runs)
          for (uint32_t k = 0; k < run.count; ++k) {
            std::pop_heap(A.begin(), A.end(), later);
            A.back() += run.cost16;
            std::push_heap(A.begin(), A.end(), later);
          }
        return A.empty() ? 0.0 : double(*std::max_element(A.begin(), A.end()));
      };
      double best = makespan(1.0);
      for (double mult : {1.125, 1.25, 1.375, 1.5}) {
        if (count_items(mult) == N) continue;  // the same plan as mult 1
        const double t = makespan(mult);
        if (t < best * 0.98) {
          best = t;
          reg_mult = mult;
        }
      }
    }
  }
  // Tiles come in runs of one row count: the split length is computed once per run.
  int last_rows = -1;
  int32_t mk = 0;
  int64_t n_parts = 0;
  for (const Tile& tl : tiles) {
    const int n = std::max(0, tl.ke - tl.k0);
    const int rows = tl.n_q * g;
    const bool t = is_tc(rows);
    const int64_t tile_keys = t ? PKV_TC_TILE_KEYS : PKV_TILE_KEYS;
    if (rows != last_rows) {
      mk = max_keys_for(rows, t, t ? 1.0 : reg_mult);
      last_rows = rows;
    }
    int32_t nseg;
    int64_t seg;
    split(n, mk, tile_keys, nseg, seg);
    const uint64_t w16 = weight16(rows);
    const int32_t gp = sc.group_of[tl.seq] >= 0 ? int32_t(sc.member_part[tl.seq]) : -1;
    if (nseg == 1 && gp < 0) {
      pieces.push_back({tl.seq, tl.q_begin, tl.n_q, tl.k0, tl.ke, tl.pos0, -1, 0, uint64_t(n) * w16, t});
      continue;
    }
    Merge mg{tl.q_begin, tl.n_q, gp, gp >= 0 ? sc.member_stride[tl.seq] : 0, int32_t(pieces.size()), nseg};
    // Partial rows of the tile's pieces, h heads an item: head hh, piece p at
    // base + ((hh / h) * nseg + p) * h * rows + (hh % h) * rows.
    const int64_t base = part_rows, hr = int64_t(heads_of(t)) * rows;
    int p = 0;
    for (int64_t k0 = tl.k0; k0 < tl.ke; k0 += seg, ++p) {
      const int k1 = int(std::min<int64_t>(tl.ke, k0 + seg));
      pieces.push_back({tl.seq, tl.q_begin, tl.n_q, int32_t(k0), k1, tl.pos0, int32_t(base + int64_t(p) * hr),
                        int32_t(int64_t(nseg) * hr), uint64_t(k1 - k0) * w16, t});
    }
    part_rows += int64_t(nseg) * rows * Hkv;
    n_parts += int64_t(nseg + (gp >= 0 ? 1 : 0)) * Hkv;
    merges.push_back(mg);
    if (part_rows > INT32_MAX) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: too many partial rows");
  }
  if (part_rows > INT32_MAX) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: too many partial rows");
  if (pieces.size() >= (size_t(1) << 20) || pieces.size() * size_t(Hkv) >= (size_t(1) << 26))
    return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: too many work items");

  size_t n_tc_pieces = 0;
  for (const Piece& pc : pieces) n_tc_pieces += pc.tc ? 1 : 0;
  const int64_t n_tc = int64_t(n_tc_pieces) * Hkv;
  const int64_t n_items = n_tc + int64_t(pieces.size() - n_tc_pieces) * (Hkv / hpi);
  const int64_t n_reduce = int64_t(merges.size()) * Hkv;

  const uint64_t items_off = sizeof(PkvPlanHeader);
  const uint64_t tc_items_off = items_off + uint64_t(n_items - n_tc) * sizeof(PkvItem);
  const uint64_t reduce_off = items_off + uint64_t(n_items) * sizeof(PkvItem);
  const uint64_t parts_off = reduce_off + uint64_t(n_reduce) * sizeof(PkvReduce);
  const uint64_t rows_off = parts_off + uint64_t(n_parts) * sizeof(int32_t);
  const uint64_t bytes = pkv_plan_bytes(rows_off + sc.row_tokens.size() * sizeof(int32_t));
  if (bytes > UINT32_MAX) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: plan too large");
  info->plan_bytes = bytes;
  info->workspace_bytes = pkv_workspace_layout(bytes, part_rows, D).total;
  info->num_items = int32_t(n_items);  // both lists
  info->num_reduce = int32_t(n_reduce);
  info->num_parts = int32_t(n_parts);
  info->num_partial_rows = int32_t(part_rows);
  info->num_groups = n_groups;
  info->num_ctas = num_ctas;
  info->num_tc_items = int32_t(n_tc);
  info->tc_num_ctas = tc_ctas;
  info->side_by_side = corun ? 1 : 0;
  info->heads_per_item = hpi;
  if (!plan) return PKV_OK;
  if (capacity < bytes) return pkv_fail(PKV_ERR_WORKSPACE, "attention_plan: capacity %zu < %llu", capacity, (unsigned long long)bytes);

  char* p = static_cast<char*>(plan);
  PkvPlanHeader h{};
  h.magic = PKV_PLAN_MAGIC;
  h.bytes = uint32_t(bytes);
  h.n_items = int32_t(n_items - n_tc);
  h.n_tc_items = int32_t(n_tc);
  h.tc_items_off = uint32_t(tc_items_off);
  h.tc_num_ctas = tc_ctas;
  h.flags = (corun ? PKV_PLAN_CORUN : 0) | (hpi == 4 ? PKV_PLAN_HEADS4 : 0);
  h.window = window;
  h.wait_limit_kcycles = req->wait_limit_kcycles;
  h.debug_flags = req->debug_flags;
  h.n_reduce = info->num_reduce;
  h.n_parts = info->num_parts;
  h.n_part_rows = info->num_partial_rows;
  h.num_seqs = S;
  h.total_q = S > 0 ? cu[S] : 0;
  h.num_q_heads = Hq;
  h.num_kv_heads = Hkv;
  h.head_dim = D;
  h.block_size = B;
  h.kv_dtype = req->kv_dtype;
  h.causal = causal ? 1 : 0;
  h.num_ctas = num_ctas;
  h.n_groups = info->num_groups;
  h.items_off = uint32_t(items_off);
  h.reduce_off = uint32_t(reduce_off);
  h.parts_off = uint32_t(parts_off);
  h.rows_off = uint32_t(rows_off);
  h.n_rows = int32_t(sc.row_tokens.size());
  std::memcpy(p, &h, sizeof(h));
  // Items: pieces heaviest first, each expanded over the KV heads (in fours on a four-head plan's
  // decode-tile list: item j takes heads 4j .. 4j + 3 and the rows of head 4j).
  PkvItem* items = reinterpret_cast<PkvItem*>(p + items_off);
  order_pieces(pieces, sc.keys, sc.tmp);
  for (size_t i = 0; i < pieces.size(); ++i) {
    const Piece& pc = pieces[size_t(sc.keys[i] & 0xFFFFF)];
    const int nh = heads_of(pc.tc);
    for (int j = 0; j < Hkv / nh; ++j)
      *items++ = PkvItem{pc.seq, j * nh, pc.q_begin, pc.n_q, pc.k_begin, pc.k_end, pc.pos0,
                         pc.part0 == -1 ? -1 : pc.part0 + j * pc.part_stride};
  }
  // Merges and their part lists, per tile and KV head: the group part first, then the pieces.
  PkvReduce* reds = reinterpret_cast<PkvReduce*>(p + reduce_off);
  int32_t* parts = reinterpret_cast<int32_t*>(p + parts_off);
  int32_t np = 0;
  for (const Merge& mg : merges) {
    for (int hh = 0; hh < Hkv; ++hh) {
      const int32_t begin = np;
      if (mg.group_part0 >= 0) parts[np++] = mg.group_part0 + hh * mg.group_stride;
      for (int k = 0; k < mg.n_pieces; ++k) {
        const Piece& pc = pieces[size_t(mg.first_piece + k)];
        const int nh = heads_of(pc.tc);
        parts[np++] = pc.part0 + (hh / nh) * pc.part_stride + (hh % nh) * pc.n_q * g;
      }
      *reds++ = PkvReduce{mg.q_begin, mg.n_q, hh, begin, np - begin, {0, 0, 0}};
    }
  }
  // The listed query tokens of group tiles, then zeros: alignment padding and the work counters.
  if (!sc.row_tokens.empty())
    std::memcpy(p + rows_off, sc.row_tokens.data(), sc.row_tokens.size() * sizeof(int32_t));
  const uint64_t used = rows_off + sc.row_tokens.size() * sizeof(int32_t);
  std::memset(p + used, 0, bytes - used);
  return PKV_OK;
}
