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
//   2. cuts every (sequence, query tile, KV head) into key ranges small enough
//      that the persistent CTAs finish together, weighting a tile by its rows
//      (compute) and keys (bytes);
//   3. emits the merges that combine split ranges (and group tiles) per row.
// On 16-bit pools tiles of more than 16 rows (prefill chunks, shared-prefix
// groups) go to a second list served by the tcgen05 kernel, 128 rows a tile,
// and are split and balanced over that kernel's CTAs on their own.  Items are
// ordered heaviest first within each list; CTAs pull them from an atomic
// counter.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <functional>
#include <queue>
#include <vector>

#include "internal.h"
#include "plan_format.h"

namespace {

struct Unit {
  int seq, kv_head, q_begin, n_q, k_begin, k_end, pos0, group_part;
  double weight;
};

struct Seg {
  PkvItem it;
  double cost;
  bool tc;  // tensor-memory list
};

// Register-tile items first, then tensor-memory items; heaviest first within each list, ties in
// creation order (the order a stable sort by cost would keep).  A cost is keys x max(1, rows/16),
// so c = 16 x cost is an integer (clamped to 32 bits past 2^25 keys).  Each item gets the key
// [list bit][c_max - c, `bits` wide][creation index, 20 bits] (the planner refuses 2^20 items or
// more), and a stable least-significant-digit radix sort over the bits above the index, in
// 11-bit digits, orders them: the indices start ascending and stability keeps ties that way.
void order_segments(const std::vector<Seg>& segs, std::vector<uint64_t>& keys, std::vector<uint64_t>& tmp) {
  const size_t n = segs.size();
  keys.resize(n);
  tmp.resize(n);
  uint64_t c_max = 0;
  for (size_t i = 0; i < n; ++i) {
    keys[i] = std::min<uint64_t>(uint64_t(segs[i].cost * 16.0 + 0.5), 0xFFFFFFFFull);
    c_max = std::max(c_max, keys[i]);
  }
  int bits = 0;
  while (bits < 32 && (c_max >> bits) != 0) ++bits;
  for (size_t i = 0; i < n; ++i)
    keys[i] = (((uint64_t(segs[i].tc) << bits) | (c_max - keys[i])) << 20) | uint64_t(i);
  if (n < 2) return;
  uint32_t count[2048];
  for (int shift = 20; shift < 21 + bits; shift += 11) {
    std::memset(count, 0, sizeof(count));
    for (size_t i = 0; i < n; ++i) ++count[(keys[i] >> shift) & 2047];
    if (count[(keys[0] >> shift) & 2047] == n) continue;  // one digit value: order unchanged
    uint32_t sum = 0;
    for (int d = 0; d < 2048; ++d) { const uint32_t c = count[d]; count[d] = sum; sum += c; }
    for (size_t i = 0; i < n; ++i) tmp[count[(keys[i] >> shift) & 2047]++] = keys[i];
    keys.swap(tmp);
  }
}

double row_weight(int rows) { return rows <= 16 ? 1.0 : rows / 16.0; }

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

  // 1. Shared-prefix groups.
  struct Group { int first, last, tokens; };
  std::vector<Group> groups;
  std::vector<int> group_of(S, -1);
  // A window would cut the shared prefix differently for every member: no groups then.
  if (req->cascade && req->block_tables && S > 1 && window == 0) {
    const int32_t* bt = req->block_tables;
    const int64_t mb = req->max_blocks;
    const int min_sh = req->min_shared_tokens > 0 ? req->min_shared_tokens : 256;
    // Blocks of a sequence every query row may see in full.
    auto usable = [&](int t) { return (causal ? L[t] - q_len(t) + 1 : L[t]) / B; };
    int s = 0;
    while (s < S) {
      if (q_len(s) < 1 || q_len(s) > QT) { ++s; continue; }
      int P = usable(s), t = s + 1;
      while (t < S && q_len(t) >= 1 && q_len(t) <= QT) {
        const int lim = std::min(P, usable(t));
        int c = 0;
        while (c < lim && bt[s * mb + c] == bt[t * mb + c]) ++c;
        if (int64_t(c) * B < min_sh) break;
        P = c;
        ++t;
      }
      if (t - s >= 2 && int64_t(P) * B >= min_sh) {
        for (int m = s; m < t; ++m) group_of[m] = int(groups.size());
        groups.push_back({s, t - 1, P * B});
        s = t;
      } else {
        ++s;
      }
    }
  }

  std::vector<Seg> segs;
  std::vector<PkvReduce> reds;
  std::vector<int32_t> parts;
  segs.reserve(size_t(S) * Hkv * 2 + 64);
  reds.reserve(size_t(S) * Hkv);
  parts.reserve(size_t(S) * Hkv * 2);
  int64_t part_rows = 0;
  // Partial row of each (group member, KV head) inside its group tile.
  std::vector<int64_t> gpart(groups.empty() ? 0 : size_t(S) * Hkv, -1);
  double total_cost[2] = {0, 0};  // register-tile list, tensor-memory list
  for (const Group& G : groups) {
    int a = G.first;
    while (a <= G.last) {
      int b = a, n = q_len(a);
      while (b + 1 <= G.last && n + q_len(b + 1) <= QT) n += q_len(++b);
      for (int h = 0; h < Hkv; ++h) {
        PkvItem it{G.first, h, cu[a], n, 0, G.tokens, -1, int32_t(part_rows)};
        for (int m = a; m <= b; ++m) gpart[size_t(m) * Hkv + h] = part_rows + int64_t(cu[m] - cu[a]) * g;
        part_rows += int64_t(n) * g;
        const double c = double(G.tokens) * row_weight(n * g);
        total_cost[is_tc(n * g)] += c;
        segs.push_back({it, c, is_tc(n * g)});
      }
      a = b + 1;
    }
  }

  // 2. Units of work.
  std::vector<Unit> units;
  units.reserve(size_t(S) * Hkv);
  for (int s = 0; s < S; ++s) {
    const int ql = q_len(s);
    if (ql == 0) continue;
    const int kb = group_of[s] >= 0 ? groups[group_of[s]].tokens : 0;
    for (int i0 = 0; i0 < ql; i0 += QT) {
      const int n = std::min(QT, ql - i0);
      const int ke = causal ? L[s] - ql + i0 + n : L[s];
      const int pos0 = causal ? L[s] - ql + i0 : -1;
      // Under a window the tile's first row sees keys from pos0 - window + 1 on; the range starts
      // there, rounded down to 128 keys (the kernels' tile alignment), and rows mask the rest.
      const int k0 = window > 0 ? std::max(kb, int(std::max(0, pos0 - window + 1) / 128 * 128)) : kb;
      for (int h = 0; h < Hkv; ++h) {
        const int gp = group_of[s] >= 0 ? int(gpart[size_t(s) * Hkv + h]) : -1;
        Unit u{s, h, cu[s] + i0, n, k0, ke, pos0, gp, row_weight(n * g)};
        total_cost[is_tc(n * g)] += double(std::max(0, ke - k0)) * u.weight;
        units.push_back(u);
      }
    }
  }

  // 3. Key-range split and merges.
  const double target[2] = {total_cost[0] / (double(num_ctas) * 2.0), total_cost[1] / (double(tc_ctas) * 2.0)};
  // Longest key range of one item of a unit's list; the automatic length (about two items per
  // CTA) is scaled by `mult`.
  auto max_keys_for = [&](const Unit& u, bool t, double mult) -> int32_t {
    const int64_t tile_keys = t ? PKV_TC_TILE_KEYS : PKV_TILE_KEYS;
    int64_t max_keys;
    if (req->kv_split < 0) max_keys = INT32_MAX;
    else if (req->kv_split > 0) max_keys = round_up(req->kv_split, tile_keys);
    else max_keys = std::max<int64_t>(std::max<int64_t>(256, 2 * tile_keys),
                                      round_up(int64_t(std::ceil(target[t] * mult / u.weight)), tile_keys));
    return int32_t(std::min<int64_t>(max_keys, INT32_MAX / 2));
  };
  // Tail check of the register-tile list.  The CTAs take items heaviest first from a counter, so
  // when the item count only just passes a multiple of the CTA count (a batch of equal long
  // ranges split into equal pieces), a few CTAs run one extra round while the rest idle.  Then
  // longer pieces are tried, and the one with the shortest simulated schedule (the greedy
  // assignment the counter produces, constant per-CTA speed) is kept if it is 2 % shorter.
  double reg_mult = 1.0;
  if (req->kv_split == 0) {
    std::vector<double> costs;
    auto list_costs = [&](double mult) {
      costs.clear();
      for (const Seg& s : segs)
        if (!s.tc) costs.push_back(s.cost);  // shared-prefix group items, never split
      int last = -1;
      int32_t m = 0;
      for (const Unit& u : units) {
        const int rows = u.n_q * g;
        if (is_tc(rows)) continue;
        if (rows != last) {
          m = max_keys_for(u, false, mult);
          last = rows;
        }
        const int n = std::max(0, u.k_end - u.k_begin);
        if (n == 0) continue;
        const uint32_t nseg = (uint32_t(n) + uint32_t(m) - 1u) / uint32_t(m);
        const int64_t seg = round_up(int64_t((uint32_t(n) + nseg - 1u) / nseg), PKV_TILE_KEYS);
        for (int64_t k0 = 0; k0 < n; k0 += seg) costs.push_back(double(std::min<int64_t>(n, k0 + seg) - k0) * u.weight);
      }
    };
    auto makespan = [&]() {
      std::sort(costs.begin(), costs.end(), std::greater<double>());
      std::priority_queue<double, std::vector<double>, std::greater<double>> load;
      for (int i = 0; i < num_ctas; ++i) load.push(0.0);
      double worst = 0.0;
      for (double c : costs) {
        const double t = load.top() + c;
        load.pop();
        load.push(t);
        worst = std::max(worst, t);
      }
      return worst;
    };
    list_costs(1.0);
    const size_t N = costs.size(), C = size_t(num_ctas);
    if (N > C && N < 4 * C && (N % C) * 4 < C) {
      double best = makespan();
      for (double mult : {1.125, 1.25, 1.375, 1.5}) {
        list_costs(mult);
        const double t = makespan();
        if (t < best * 0.98) {
          best = t;
          reg_mult = mult;
        }
      }
    }
  }
  // Units come in runs of one row count (every KV head of a tile): the split length is computed
  // once per run.
  int last_rows = -1;
  int32_t mk = 0;
  for (const Unit& u : units) {
    const int n = std::max(0, u.k_end - u.k_begin);
    const int rows = u.n_q * g;
    const bool t = is_tc(rows);
    const int64_t tile_keys = t ? PKV_TC_TILE_KEYS : PKV_TILE_KEYS;
    if (rows != last_rows) {
      mk = max_keys_for(u, t, t ? 1.0 : reg_mult);
      last_rows = rows;
    }
    const int32_t nseg = n == 0 ? 0 : int32_t((uint32_t(n) + uint32_t(mk) - 1u) / uint32_t(mk));
    if (nseg == 1 && u.group_part < 0) {
      PkvItem it{u.seq, u.kv_head, u.q_begin, u.n_q, u.k_begin, u.k_end, u.pos0, -1};
      segs.push_back({it, n * u.weight, t});
      continue;
    }
    PkvReduce r{u.q_begin, u.n_q, u.kv_head, int32_t(parts.size()), 0, {0, 0, 0}};
    if (u.group_part >= 0) parts.push_back(u.group_part);
    if (nseg > 0) {
      const int64_t seg = round_up(int64_t((uint32_t(n) + uint32_t(nseg) - 1u) / uint32_t(nseg)), tile_keys);
      for (int64_t k0 = u.k_begin; k0 < u.k_end; k0 += seg) {
        const int k1 = int(std::min<int64_t>(u.k_end, k0 + seg));
        PkvItem it{u.seq, u.kv_head, u.q_begin, u.n_q, int(k0), k1, u.pos0, int32_t(part_rows)};
        parts.push_back(int32_t(part_rows));
        part_rows += rows;
        segs.push_back({it, (k1 - k0) * u.weight, t});
      }
    }
    r.n_parts = int32_t(parts.size()) - r.parts_begin;
    reds.push_back(r);
  }
  if (part_rows > INT32_MAX) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: too many partial rows");
  if (segs.size() >= (size_t(1) << 20)) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: more than 2^20 work items");

  const int64_t n_tc = std::count_if(segs.begin(), segs.end(), [](const Seg& s) { return s.tc; });

  const uint64_t items_off = sizeof(PkvPlanHeader);
  const uint64_t tc_items_off = items_off + (segs.size() - n_tc) * sizeof(PkvItem);
  const uint64_t reduce_off = items_off + segs.size() * sizeof(PkvItem);
  const uint64_t parts_off = reduce_off + reds.size() * sizeof(PkvReduce);
  const uint64_t bytes = pkv_plan_bytes(parts_off + parts.size() * sizeof(int32_t));
  if (bytes > UINT32_MAX) return pkv_fail(PKV_ERR_UNSUPPORTED, "attention_plan: plan too large");
  info->plan_bytes = bytes;
  info->workspace_bytes = pkv_workspace_layout(bytes, part_rows, D).total;
  info->num_items = int32_t(segs.size());  // both lists
  info->num_reduce = int32_t(reds.size());
  info->num_parts = int32_t(parts.size());
  info->num_partial_rows = int32_t(part_rows);
  info->num_groups = int32_t(groups.size());
  info->num_ctas = num_ctas;
  info->num_tc_items = int32_t(n_tc);
  if (!plan) return PKV_OK;
  if (capacity < bytes) return pkv_fail(PKV_ERR_WORKSPACE, "attention_plan: capacity %zu < %llu", capacity, (unsigned long long)bytes);

  char* p = static_cast<char*>(plan);
  std::memset(p, 0, bytes);
  PkvPlanHeader h{};
  h.magic = PKV_PLAN_MAGIC;
  h.bytes = uint32_t(bytes);
  h.n_items = int32_t(segs.size() - n_tc);
  h.n_tc_items = int32_t(n_tc);
  h.tc_items_off = uint32_t(tc_items_off);
  h.tc_num_ctas = tc_ctas;
  h.window = window;
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
  std::memcpy(p, &h, sizeof(h));
  PkvItem* items = reinterpret_cast<PkvItem*>(p + items_off);
  std::vector<uint64_t> order, scratch;
  order_segments(segs, order, scratch);
  for (size_t i = 0; i < segs.size(); ++i) items[i] = segs[size_t(order[i] & 0xFFFFF)].it;
  if (!reds.empty()) std::memcpy(p + reduce_off, reds.data(), reds.size() * sizeof(PkvReduce));
  if (!parts.empty()) std::memcpy(p + parts_off, parts.data(), parts.size() * sizeof(int32_t));
  return PKV_OK;
}
