// Work-list format shared by the host planner and the attention kernels.
//
// A plan is one contiguous buffer: header, items, tensor-memory items, merges,
// part list.  The host builds it (plan.cpp), paged_attention copies it into
// the device workspace, and the CTAs of each persistent kernel pull items
// from their own list.
#pragma once
#include <stdint.h>

#define PKV_PLAN_MAGIC 0x314e4c50u  // "PLN1"

// Rows of one work item (query tokens x the Hq/Hkv query heads of one KV
// head) for the register-tile kernels.
#define PKV_TILE_ROWS 64
// Keys per pipeline stage of the register-tile kernels.
#define PKV_TILE_KEYS 64
// Tensor-memory items (16-bit pools; fp8 pools of head_dim 128): more than PKV_DECODE_ROWS and at most
// PKV_TILE_ROWS_TC rows (one tensor-memory lane per row), keys in tiles of
// PKV_TC_TILE_KEYS; a split key range starts on a multiple of that.
#define PKV_DECODE_ROWS 16
#define PKV_FP4_ROWS 8     /* rows per tile on NVFP4 pools (one register tile of query rows) */
#define PKV_TILE_ROWS_TC 128
#define PKV_TC_TILE_KEYS 128
// Limit of every pipeline wait of the attention kernels when the plan gives none, in SM cycles
// (2.0 s at 1965 MHz, about 3 s at 1.3 GHz).
#define PKV_DEFAULT_WAIT_CYCLES 4000000000ll

struct PkvPlanHeader {
  uint32_t magic;
  uint32_t bytes;        // whole plan, header included
  int32_t n_items;
  int32_t n_reduce;
  int32_t n_parts;
  int32_t n_part_rows;
  int32_t num_seqs;
  int32_t total_q;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t kv_dtype;
  int32_t causal;
  int32_t num_ctas;
  int32_t n_groups;
  uint32_t items_off;    // byte offsets from the start of the plan
  uint32_t reduce_off;
  uint32_t parts_off;
  int32_t n_tc_items;    // tensor-memory items (attn_tc kernel), after the others
  uint32_t tc_items_off;
  int32_t tc_num_ctas;   // CTAs planned for the tensor-memory kernel
  int32_t window;        // limited attention window in positions; 0 = none
  int32_t wait_limit_kcycles;  // limit on every pipeline wait, thousands of SM cycles; 0 = default
  int32_t debug_flags;   // PKV_DEBUG_* (0 in normal use)
  int32_t flags;         // PKV_PLAN_* bits
  uint32_t rows_off;     // listed query tokens of group tiles (int32 each)
  int32_t n_rows;
  int32_t pad[4];        // header is 128 bytes
};
static_assert(sizeof(PkvPlanHeader) == 128, "plan header size");
// The two item lists run side by side: the tcgen05 kernel is launched first on tc_num_ctas CTAs
// (one an SM) and the decode-tile kernel beside it on num_ctas CTAs (the other SMs).  Without it
// the decode-tile kernel runs first and the tcgen05 kernel takes the SMs it frees.
#define PKV_PLAN_CORUN 0x1
// Every item of the decode-tile list covers four consecutive KV heads, kv_head .. kv_head + 3
// (kv_head a multiple of 4), with at most PKV_HEADS4_ROWS rows per head; head kv_head + w of it
// writes its partial rows at part_row + w * n_q * g.  Only the TMA-fed decode kernel takes such
// plans: each of its four consumer warps runs one of the heads over the whole key range.
#define PKV_PLAN_HEADS4 0x2
#define PKV_HEADS4_ROWS 8

// One CTA-sized piece of work: rows [q_begin, q_begin + n_q) x the g query
// heads of kv_head, against keys [k_begin, k_end) read through the block-table
// row of `seq`.  Row r of the tile is query token q_begin + r / g, head
// kv_head * g + r % g.  With pos0 >= 0 the tile is causal: token q_begin + i
// sits at position pos0 + i and sees keys < pos0 + i + 1.  part_row < 0 writes
// the final output; otherwise the normalised partial state goes to partial rows
// part_row .. part_row + n_q * g - 1.  pos0 <= -2 (shared-prefix group tiles
// of the tensor-memory list, which are not causal): the tile's query tokens are not the run
// q_begin .. but listed, token i at row_tokens[-2 - pos0 + i] (q_begin is the first of them).
struct PkvItem {
  int32_t seq;
  int32_t kv_head;
  int32_t q_begin;
  int32_t n_q;
  int32_t k_begin;
  int32_t k_end;
  int32_t pos0;
  int32_t part_row;
};
static_assert(sizeof(PkvItem) == 32, "item size");

// Output rows [q_begin, q_begin + n_q) x heads of kv_head, merged from the
// partial states listed in parts[parts_begin .. parts_begin + n_parts): entry
// p names the partial row holding row 0 of this tile.
struct PkvReduce {
  int32_t q_begin;
  int32_t n_q;
  int32_t kv_head;
  int32_t parts_begin;
  int32_t n_parts;
  int32_t pad[3];
};
static_assert(sizeof(PkvReduce) == 32, "reduce size");

// The plan buffer ends in a 256-byte block of zeros, 256-byte aligned: the
// kernels' work counters (the register-tile kernel's at +0, the tensor-memory
// kernel's at +128).  Uploading the plan therefore also clears the counters.
#define PKV_PLAN_COUNTER_BYTES 256
static inline uint64_t pkv_align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }
// Plan bytes for a body (header, items, merges, parts) of `body` bytes.
static inline uint64_t pkv_plan_bytes(uint64_t body) { return pkv_align256(body) + PKV_PLAN_COUNTER_BYTES; }

// Device workspace layout: [plan copy with its counters][partial o][partial lse].
struct PkvWorkspaceLayout {
  uint64_t plan_off, counter_off, counter_bytes, part_o_off, part_lse_off, total;
};
static inline PkvWorkspaceLayout pkv_workspace_layout(uint64_t plan_bytes, int64_t n_part_rows, int head_dim) {
  PkvWorkspaceLayout L;
  L.plan_off = 0;
  L.counter_off = plan_bytes - PKV_PLAN_COUNTER_BYTES;
  L.counter_bytes = PKV_PLAN_COUNTER_BYTES;
  L.part_o_off = pkv_align256(plan_bytes);
  L.part_lse_off = pkv_align256(L.part_o_off + uint64_t(n_part_rows) * head_dim * 4);
  L.total = pkv_align256(L.part_lse_off + uint64_t(n_part_rows) * 4);
  return L;
}
