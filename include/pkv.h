/*
 * pkv.h - C ABI of libpkv.so: attention over a paged KV cache on B200 (sm_100a).
 *
 * The operations follow the pages on NVIDIA TensorRT-LLM this library is built
 * from:
 *   - the KV cache is a pool of fixed-size token blocks, a request reaches its
 *     blocks through a per-request block table, and the block size is a power
 *     of two greater than one ("NVIDIA TensorRT-LLM详解", gentlecold.top, §9
 *     "KV cache系统");
 *   - new tokens' K/V are written into their pages through a page-table lookup
 *     (TensorRT-LLM concept explainer, compassingai.com, "技术原理"; deep dive
 *     §2, decode writes the new token's KV);
 *   - one batch packs context (prefill) requests before generation (decode)
 *     requests, without padding, and a long prompt is processed in chunks that
 *     attend to everything cached so far plus themselves (deep dive §6
 *     "In-flight batching", §8 "Chunked prefill");
 *   - the cache may be stored as fp8 or as NVFP4 (deep dive §13 "量化：FP8、FP4与
 *     KV cache dtype": KvCacheConfig(dtype="fp8") and dtype="nvfp4").
 * The attention itself is softmax(scale * q K^T) V with grouped-query heads:
 * query head h reads KV head h / (Hq / Hkv).
 *
 * Conventions shared by every call:
 *   - Memory: every pointer named "device" is CUDA device memory owned by the
 *     caller; "host" pointers are host memory owned by the caller.  The library
 *     never allocates or frees memory and never synchronises the stream.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued in call order on that stream.
 *   - Synchronous errors: an invalid argument returns a nonzero pkv_status at
 *     once and enqueues nothing.  PKV_ERR_CUDA reports a failed launch or copy;
 *     pkv_last_error() gives a message for the calling thread.
 *   - Asynchronous errors: a block id outside [0, num_blocks), a logical block
 *     beyond the table row, or a plan that does not match the lengths on the
 *     device is recorded by OR-ing a PKV_DEV_* bit into *dev_status (device
 *     int32, zeroed by the caller, may be NULL).  kv_append and copy_block_prefix
 *     skip the offending rows; paged_attention skips work items that do not fit
 *     the device lengths and reads the keys of an out-of-range block as zeros
 *     (no memory outside the pool is read; the affected rows' outputs are not
 *     meaningful, every other row is unaffected).  No kernel traps.
 *   - Pool layout (row-major):
 *       pool[num_blocks][num_layers][2][num_kv_heads][block_size][head_dim]
 *     index 0 of the "2" axis is K, 1 is V; each (block, layer, K|V, head) is
 *     one contiguous run of block_size * head_dim elements.  An NVFP4 pool
 *     keeps the same order with a different run: block_size rows of
 *     head_dim / 2 bytes of packed E2M1 codes (dimension 2i in the low nibble
 *     of byte i, 2i+1 in the high nibble), then block_size rows of
 *     head_dim / 16 bytes of E4M3 block scales (byte j scales dimensions
 *     16j .. 16j+15 of its row): block_size * head_dim * 9 / 16 bytes per run.
 *   - Token p of sequence s lives in physical block block_tables[s][p / B] at
 *     slot p % B.  Block tables are int32 [num_seqs][max_blocks] (row stride
 *     max_blocks); unused entries are ignored.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_ABI_VERSION 4

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1, /* null pointer, bad shape or dtype, lengths out of range */
  PKV_ERR_UNSUPPORTED = 2, /* valid but not built: e.g. head_dim outside {64, 128} */
  PKV_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  PKV_ERR_WORKSPACE = 4,   /* caller buffer smaller than required */
  PKV_ERR_PLAN = 5         /* plan buffer corrupt or made for other shapes */
} pkv_status;

typedef enum pkv_dtype {
  PKV_F32 = 0,
  PKV_BF16 = 1,
  PKV_F16 = 2,
  PKV_FP8_E4M3 = 3, /* OCP E4M3: bias 7, no infinities, max finite 448 */
  PKV_NVFP4 = 4     /* KV pools only: E2M1 codes (1 sign, 2 exponent, 1 mantissa bit:
                       0, 0.5, 1, 1.5, 2, 3, 4, 6) with an E4M3 scale per 16 values and a
                       float32 scale per (layer, KV head, K|V); value = code * block scale
                       * k_scale or v_scale.  head_dim 128, block_size >= 16. */
} pkv_dtype;

/* Bits OR-ed into *dev_status by kernels. */
#define PKV_DEV_BAD_BLOCK_ID 0x1      /* block table entry outside [0, num_blocks) */
#define PKV_DEV_BAD_LOGICAL_BLOCK 0x2 /* position needs a table entry beyond max_blocks */
#define PKV_DEV_PLAN_MISMATCH 0x4     /* plan item does not fit the device lengths */
#define PKV_DEV_BAD_APPEND 0x8        /* kv_append position negative */
#define PKV_DEV_TIMEOUT 0x10          /* an internal pipeline wait gave up (after the plan's wait limit: by default
                                         4e9 SM cycles, 2.0 s at 1965 MHz); results incomplete */
#define PKV_DEV_BAD_COPY 0x20         /* copy_block_prefix: token count outside [0, block_size] */

/* One layer's view of a paged pool (deep dive §9: one block holds a fixed number
 * of tokens' KV; several layers may be packed in one block). */
typedef struct pkv_cache {
  void* pool;             /* device, layout above, element type kv_dtype */
  int64_t num_blocks;     /* physical blocks in the pool */
  int32_t num_layers;     /* layers packed per block */
  int32_t layer;          /* layer this call reads or writes, 0 <= layer < num_layers */
  int32_t num_kv_heads;   /* Hkv */
  int32_t head_dim;       /* d: 64 or 128 */
  int32_t block_size;     /* B: power of two, >= 2 */
  int32_t kv_dtype;       /* pkv_dtype: F32, BF16, F16, FP8_E4M3 or NVFP4 */
  const float* k_scale;   /* device float32 [num_layers][Hkv], positive and finite; FP8_E4M3 and NVFP4 only */
  const float* v_scale;   /* device float32 [num_layers][Hkv], positive and finite; FP8_E4M3 and NVFP4 only */
} pkv_cache;

/* Library ABI version (PKV_ABI_VERSION of the build). */
PKV_API int32_t pkv_abi_version(void);

/* Static description of a status code. */
PKV_API const char* pkv_status_string(int32_t status);

/* Detail of the last error raised on the calling thread ("" if none). */
PKV_API const char* pkv_last_error(void);

/*
 * kv_append - write new tokens' K and V into their pool slots.
 *
 * Source: deep dive §2 (decode writes each new token's KV), §8 (a prefill chunk
 * appends its KV before the next chunk), concept explainer "技术原理" (page-table
 * lookup on KV writes).
 *
 * k_new, v_new: device [total_new][Hkv][head_dim] of in_dtype, packed by
 *   sequence: sequence s owns rows cu_new[s] .. cu_new[s+1]-1.
 * cu_new: device int32 [num_seqs+1], cu_new[0] = 0, nondecreasing,
 *   cu_new[num_seqs] = total_new (total_new also passed by value for the grid).
 * start_pos: device int32 [num_seqs]: position of sequence s's first new token;
 *   row cu_new[s]+i goes to position start_pos[s]+i.
 * block_tables: device int32 [num_seqs][max_blocks].
 * in_dtype: must equal cache->kv_dtype for F32/BF16/F16 pools.  For an
 *   FP8_E4M3 pool it is F32, BF16 or F16 and each value x is stored as the
 *   E4M3 code of the float32 quotient x / scale (IEEE division), rounded to
 *   nearest even, finite overflow saturated to +-448, with scale =
 *   k_scale[layer][h] for K and v_scale[layer][h] for V.  For an NVFP4 pool it
 *   is F32, BF16 or F16 (finite values); each row's 16-value group x with
 *   global scale g = k_scale[layer][h] (K) or v_scale[layer][h] (V) is stored,
 *   all in float32 with IEEE rounding, as: a = max |x_i|; block scale code
 *   c = E4M3(a / (6 * g)) (nearest even, saturating); s = value of c; codes
 *   E2M1(x_i / (s * g)), nearest even, saturating to +-6, the sign kept (all
 *   codes 0 when s = 0).
 * Errors: INVALID_ARG for bad shapes/dtypes/null pointers.  Asynchronously,
 *   rows whose block id is out of range are not written (PKV_DEV_BAD_BLOCK_ID,
 *   PKV_DEV_BAD_LOGICAL_BLOCK, PKV_DEV_BAD_APPEND).
 * Stream-ordered; reads no memory after the kernel completes.
 */
PKV_API pkv_status pkv_kv_append(const pkv_cache* cache, const void* k_new, const void* v_new, int32_t in_dtype,
                         const int32_t* cu_new, const int32_t* start_pos, const int32_t* block_tables,
                         int32_t max_blocks, int32_t num_seqs, int32_t total_new, int32_t* dev_status,
                         void* stream);

/*
 * copy_block_prefix - copy the first tokens of pool blocks into other blocks.
 *
 * Source: deep dive §11 (partial reuse: when a new request matches only part of
 * a cached block, copy_on_partial_reuse copies the matched tokens of that block
 * into a new block, so that several requests can reuse the same block
 * partially while each appends its own tokens after the copy).
 *
 * For i in [0, count): slots 0 .. n_tokens[i]-1 of block src_blocks[i] are
 * copied into the same slots of block dst_blocks[i], for every layer, K and
 * V, and every KV head; slots n_tokens[i] .. block_size-1 of the destination
 * are left as they were.  n_tokens[i] = block_size copies the whole block.
 * src_blocks, dst_blocks, n_tokens: device int32 [count].
 * A destination must not be the source or destination of another copy of the
 * same call (such copies race); src == dst is a no-op.
 * Errors: INVALID_ARG for bad shapes / null pointers.  Asynchronously, copies
 *   with a block id outside [0, num_blocks) (PKV_DEV_BAD_BLOCK_ID) or a token
 *   count outside [0, block_size] (PKV_DEV_BAD_COPY) are skipped.
 * Stream-ordered; bit-exact (a byte copy, any pool dtype; for NVFP4 pools, head_dim
 *   128, the slots' codes and their block scales).
 */
PKV_API pkv_status pkv_copy_block_prefix(const pkv_cache* cache, const int32_t* src_blocks,
                                         const int32_t* dst_blocks, const int32_t* n_tokens, int32_t count,
                                         int32_t* dev_status, void* stream);

/*
 * Planning request for one paged_attention call (a batch of sequences).
 *
 * Sequence s processes q_len = cu_q_lens[s+1] - cu_q_lens[s] query tokens this
 * step (1 for decode, the chunk length for a prefill chunk, 0 = not scheduled)
 * and attends over seq_lens[s] keys, counting this step's tokens, which must
 * already be appended.  Query row j of s sits at position seq_lens[s] - q_len
 * + j; with causal != 0 it attends to keys 0..position (deep dive §8: a chunk
 * sees the cached KV plus itself), otherwise to all seq_lens[s] keys.
 */
typedef struct pkv_plan_request {
  int32_t num_seqs;
  int32_t num_q_heads;          /* Hq, a multiple of num_kv_heads */
  int32_t num_kv_heads;         /* Hkv */
  int32_t head_dim;             /* 64 or 128 (128 for NVFP4 pools) */
  int32_t block_size;           /* power of two >= 2 (>= 16 for NVFP4 pools) */
  int32_t kv_dtype;             /* pkv_dtype of the pool */
  int32_t causal;               /* 0 or 1 */
  int32_t num_ctas;             /* CTAs the launch uses (capped at what fits resident); 0 = all that
                                   fit on the current device */
  int32_t kv_split;             /* 0 = automatic split of long key ranges; >0 = max keys per work
                                   item (rounded up to 64); <0 = never split */
  int32_t cascade;              /* nonzero: group consecutive sequences whose tables share leading
                                   blocks and read those blocks once per group (needs block_tables) */
  int32_t min_shared_tokens;    /* shortest shared prefix that forms a group (0 = 256) */
  int32_t max_blocks;           /* row stride of block_tables */
  const int32_t* cu_q_lens;     /* host int32 [num_seqs+1] */
  const int32_t* seq_lens;      /* host int32 [num_seqs] */
  const int32_t* block_tables;  /* host int32 [num_seqs][max_blocks]; NULL disables cascade */
  int32_t window;               /* limited attention window (deep dive §11: tokens outside the window
                                   no longer take part in attention): query row at position p sees keys
                                   p - window < t <= p.  0 = no limit.  Needs causal; disables cascade.
                                   The plan carries it to pkv_paged_attention. */
  int32_t wait_limit_kcycles;   /* limit on every internal pipeline wait of the attention kernels, in
                                   thousands of SM cycles; 0 = the default 4e6 (4e9 cycles: 2.0 s at 1965
                                   MHz, about 3 s at 1.3 GHz).  A wait that runs out sets PKV_DEV_TIMEOUT,
                                   and the kernel stops issuing work, waits (bounded) for its own copies
                                   in flight, frees its tensor memory and exits.  >= 0. */
  int32_t debug_flags;          /* 0 in normal use.  PKV_DEBUG_WITHHOLD_LOADS: the producers of the
                                   TMA-fed decode kernel and of the tcgen05 kernel publish every work
                                   item but load no K/V tile, so every consumer wait runs out: a way to
                                   test the timeout path (with a short wait_limit_kcycles) without a
                                   fault.  Outputs are then incomplete.  Kernels without a TMA producer
                                   (block sizes below 8, 64-byte fp8 rows, fp32 pools) ignore it. */
  int32_t tc_num_ctas;          /* side by side: tiles of more than 16 rows (the tcgen05 kernel, deep dive
                                   §6/§8 prefill chunks and §10 shared-prefix group tiles) and the
                                   decode-sized tiles (the HBM stream) in one call run at the same time on
                                   disjoint SMs, the tcgen05 kernel on tc_num_ctas CTAs (one an SM) and the
                                   decode-tile kernel on num_ctas CTAs, instead of one after the other.
                                   > 0: side by side on these counts whenever the batch has both kinds of
                                   tile (num_ctas must then be > 0 too; both are capped at what fits).
                                   0: automatic, with num_ctas = 0 only: side by side when the planner's
                                   estimate of the two kernels' times says it pays, splitting the SMs of
                                   the current device between them.  < 0: never.  Plans are the same for
                                   every layer either way. */
  int32_t heads_per_item;       /* KV heads one decode-sized work item covers.  4: each item of the
                                   decode-tile list takes four consecutive KV heads of one query tile
                                   and key range, one head per consumer warp of the TMA-fed decode
                                   kernel, so a warp runs its head over the whole range and no warps'
                                   states are merged at the item's end (short key ranges: many small
                                   decode requests, shared-prefix members' own suffixes).  Needs
                                   num_kv_heads a multiple of 4, a pool the TMA-fed kernel serves
                                   (16-bit pools with block_size >= 8, fp8 pools of head_dim 128 with
                                   block_size >= 8, NVFP4 pools) and at most 8 rows per decode tile
                                   (query tokens x Hq/Hkv); else UNSUPPORTED.  1: one KV head per item.
                                   0: automatic, 4 where it applies on NVFP4 pools (instruction-bound
                                   tiles) and, on the others, where the decode tiles' key ranges are
                                   short against the per-CTA share of the batch. */
} pkv_plan_request;

#define PKV_DEBUG_WITHHOLD_LOADS 0x1

typedef struct pkv_plan_info {
  size_t plan_bytes;            /* bytes of the plan buffer */
  size_t workspace_bytes;       /* device workspace paged_attention needs with this plan */
  int32_t num_items;            /* work items (one CTA-sized tile of rows x key range each) */
  int32_t num_reduce;           /* output row groups merged from partial states */
  int32_t num_parts;            /* partial states referenced by the merges */
  int32_t num_partial_rows;     /* float32 partial rows of head_dim (+1 lse) in the workspace */
  int32_t num_groups;           /* shared-prefix groups found */
  int32_t num_ctas;             /* CTAs planned for */
  int32_t num_tc_items;         /* of num_items: tiles of more than 16 rows for the tcgen05 kernel */
  int32_t tc_num_ctas;          /* CTAs planned for the tcgen05 kernel */
  int32_t side_by_side;         /* 1: the two kernels run at the same time on disjoint SMs (num_ctas
                                   and tc_num_ctas CTAs); 0: one after the other */
  int32_t heads_per_item;       /* KV heads per item of the decode-tile list (1 or 4) */
} pkv_plan_info;

/*
 * attention_plan - host-only: split the batch into work items for one launch.
 *
 * Cuts every (sequence, KV head, query tile) into key ranges so that the work
 * spreads evenly over num_ctas CTAs, and, with cascade, finds sequences whose
 * tables share leading physical blocks (deep dive §10: prefix blocks reused
 * across requests through the radix tree) so that those keys are read once per
 * group.  The plan depends only on the lengths, the tables' sharing pattern and
 * the shapes: a runtime plans once per step and reuses the plan for every layer.
 *
 * plan: host buffer of `capacity` bytes, or NULL to query sizes only.
 * info: filled in all cases (required).
 * Returns WORKSPACE if capacity < info->plan_bytes, INVALID_ARG on bad lengths
 * (q_len > seq_len, negative values, a table row too short for seq_len, Hq not a
 * multiple of Hkv, more than 64 query heads per KV head).  Touches no GPU
 * unless num_ctas == 0.
 */
PKV_API pkv_status pkv_attention_plan(const pkv_plan_request* req, void* plan, size_t capacity, pkv_plan_info* info);

/* CTAs the attention kernel for this pool dtype, head_dim and block size keeps
 * resident on the current device (SM count x occupancy). */
PKV_API pkv_status pkv_default_num_ctas(int32_t kv_dtype, int32_t head_dim, int32_t block_size, int32_t* num_ctas);

/*
 * paged_attention - out = softmax(scale * q K^T) V over each sequence's paged K/V.
 *
 * Source: deep dive §2 (decode reads all history KV to do attention), §6 (one
 * launch serves a packed mix of prefill and decode requests), §8 (chunked
 * prefill with causal masking).  One call enqueues one persistent attention
 * kernel for the decode-sized tiles, one tcgen05 kernel for the tiles of more
 * than 16 rows of a bf16/f16 pool or an fp8 pool of head_dim 128 (when the plan
 * has such tiles) and, when the plan split a key range, one merge kernel (the
 * same merge pkv_split_kv_reduce performs), in that order on `stream`; a plan
 * made side by side (pkv_plan_info.side_by_side) enqueues the tcgen05 kernel
 * first and the decode-tile kernel beside it, on the SMs it leaves free.  A plan
 * with four-head items (pkv_plan_info.heads_per_item 4) runs the decode-tile
 * kernel's four-head variant: one consumer warp per KV head of an item.
 *
 * q: device [total_q][num_q_heads][head_dim], q_dtype F32 (F32 pools only),
 *   BF16 (BF16, FP8 or NVFP4 pools) or F16 (F16, FP8 or NVFP4 pools).
 *   total_q = cu_q_lens[num_seqs].  NVFP4 pools: head_dim 128, block_size >= 16,
 *   at most 8 query heads per KV head (else UNSUPPORTED, from the planner too).
 * cu_q_lens, seq_lens: device int32 copies of the arrays the plan was made from.
 * block_tables: device int32 [num_seqs][max_blocks].
 * softmax_scale: scale on q.k (typically 1/sqrt(head_dim)), positive and finite;
 *   causal as planned.  fp8 and NVFP4 scales must be positive.
 * plan: host buffer from pkv_attention_plan for these shapes.  It is staged in
 *   the workspace on `stream`: a page-locked plan by a kernel that reads it
 *   through its device alias (launched as a programmatic dependent of the work
 *   ahead of it), any other plan by cudaMemcpyAsync.  Keep it unchanged until
 *   the staging has run.
 * out: device [total_q][num_q_heads][head_dim] in q_dtype.
 * out_lse: device float32 [total_q][num_q_heads] natural-log sum of exp(scores)
 *   per row, or NULL.
 * q, out and the pool must be 16-byte aligned.
 * workspace: device, >= info.workspace_bytes, 256-byte aligned.
 * Errors: INVALID_ARG/UNSUPPORTED/PLAN/WORKSPACE synchronously; PKV_DEV_* bits
 *   asynchronously (skipped rows are left unwritten).
 */
PKV_API pkv_status pkv_paged_attention(const pkv_cache* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                               const int32_t* cu_q_lens, const int32_t* seq_lens, const int32_t* block_tables,
                               int32_t max_blocks, int32_t num_seqs, float softmax_scale, int32_t causal,
                               const void* plan, void* out, float* out_lse, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * paged_attention_timed - pkv_paged_attention that also records two CUDA
 * events (cudaEvent_t, created by the caller; either may be NULL) on `stream`:
 * kernels_begin right before the attention kernels and kernels_end right after
 * them, before the merge of split key ranges.  With events created for timing,
 * cudaEventElapsedTime gives the attention kernels' own duration (also inside a
 * captured graph).  Arguments, results and errors are otherwise those of
 * pkv_paged_attention.
 */
PKV_API pkv_status pkv_paged_attention_timed(const pkv_cache* cache, const void* q, int32_t q_dtype,
                               int32_t num_q_heads, const int32_t* cu_q_lens, const int32_t* seq_lens,
                               const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                               float softmax_scale, int32_t causal, const void* plan, void* out, float* out_lse,
                               void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream,
                               void* kernels_begin, void* kernels_end);

/*
 * split_kv_reduce - merge partial softmax states computed over disjoint key sets.
 *
 * The pages do not describe split-KV; this is the exact identity that splitting
 * a softmax over key ranges obeys.  For each row r:
 *   M = max_i lse[i][r];  w_i = exp(lse[i][r] - M);
 *   out[r] = sum_i w_i o[i][r] / sum_i w_i;  out_lse[r] = M + ln(sum_i w_i).
 * A part with lse = -inf (no keys) has weight 0; a row whose parts are all
 * empty gets out = 0 and out_lse = -inf.
 *
 * partial_o: device float32 [n_split][rows][head_dim], each part normalised.
 * partial_lse: device float32 [n_split][rows], natural log.
 * out: device [rows][head_dim] in out_dtype (F32, BF16 or F16).
 * out_lse: device float32 [rows] or NULL.
 */
PKV_API pkv_status pkv_split_kv_reduce(const float* partial_o, const float* partial_lse, int32_t n_split, int64_t rows,
                               int32_t head_dim, void* out, int32_t out_dtype, float* out_lse, void* stream);

/*
 * stream_read - a plain read-only stream over device memory (a measurement aid).
 *
 * Decode attention reads every cached K/V byte once per step (deep dive §2:
 * decode reads all history KV), so the fastest plain read of HBM is the
 * practical ceiling its bandwidth is judged against.  This reads `bytes`
 * bytes at `src` once and XOR-folds them into *sink (device uint32, any
 * initial value) so that no load is dead.
 * mode 0: every thread issues 16-byte non-caching loads over a grid-strided
 *   range (4 CTAs of 512 threads per SM);
 * mode 1: one elected thread per CTA copies 32 KB chunks into a 4-stage
 *   shared-memory ring with 1-D bulk async copies counted on mbarriers, as the
 *   attention kernels' TMA producers do (one CTA per SM, no multicast).
 * src and bytes: multiples of 16.  dev_status: PKV_DEV_TIMEOUT if a ring wait
 *   of mode 1 gives up (may be NULL).  Stream-ordered; allocates nothing.
 */
PKV_API pkv_status pkv_stream_read(const void* src, size_t bytes, int32_t mode, uint32_t* sink,
                                   int32_t* dev_status, void* stream);

/*
 * paged_attention_noalloc - paged_attention for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it exists for callers that are
 * handed only input and output buffers and may not allocate device memory
 * themselves (a plug-in inside a host framework, an allocator-free runtime, or
 * code whose device memory budget is fixed before it runs).  Arguments and
 * results are those of pkv_paged_attention without the workspace: the scratch
 * (plan copy, work counter, split partials) lives in one device array of
 * PKV_NOALLOC_SCRATCH_BYTES built into the library, which every GPU that loads
 * the library holds until the process exits.
 *   - A plan needing more scratch than that returns PKV_ERR_WORKSPACE.
 *   - The first call on a device looks up the array's address on that device;
 *     make it outside any stream capture.  After the device's context changes
 *     (cudaDeviceReset, a context destroyed and created again) the array may
 *     move: the next call notices the new context and looks the address up
 *     again, so make that call outside stream capture as well.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents (the work counters are cleared by each call's plan upload).  Calls that
 *     overlap on the GPU race; order them on one stream.
 *   - Allocates and frees nothing.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (32ull << 20)
PKV_API pkv_status pkv_paged_attention_noalloc(const pkv_cache* cache, const void* q, int32_t q_dtype,
                                       int32_t num_q_heads, const int32_t* cu_q_lens, const int32_t* seq_lens,
                                       const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                       float softmax_scale, int32_t causal, const void* plan, void* out,
                                       float* out_lse, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
