// C ABI: argument checks, plan upload and launches of paged_attention, plus the
// small shared entry points (version, status strings, error detail, occupancy).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>

#include "attn_args.h"
#include "internal.h"
#include "plan_format.h"

namespace {
thread_local char g_last_error[512] = "";
}

pkv_status pkv_fail(pkv_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

extern "C" int32_t pkv_abi_version(void) { return PKV_ABI_VERSION; }

extern "C" const char* pkv_status_string(int32_t status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_WORKSPACE: return "buffer too small";
    case PKV_ERR_PLAN: return "plan does not match the call";
    default: return "unknown status";
  }
}

extern "C" const char* pkv_last_error(void) { return g_last_error; }

namespace pkv {
// SM count x occupancy, cached per (device, kernel).
int resident_ctas(const AttnKernel& k) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, k.fn});
  if (it != cache.end()) return it->second;
  int sms = 0, per_sm = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess && k.smem > 48 * 1024)
    e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
  if (e == cudaSuccess && k.smem > 48 * 1024 && k.fn_heads4)
    e = cudaFuncSetAttribute(k.fn_heads4, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.fn, k.threads, k.smem);
  if (e != cudaSuccess) return -1;
  const int n = std::max(1, sms * std::max(1, per_sm));
  cache[{dev, k.fn}] = n;
  return n;
}
}  // namespace pkv

extern "C" pkv_status pkv_default_num_ctas(int32_t kv_dtype, int32_t head_dim, int32_t block_size, int32_t* num_ctas) {
  if (!num_ctas) return pkv_fail(PKV_ERR_INVALID_ARG, "default_num_ctas: null output");
  pkv::AttnKernel k;
  const int q_dtype = kv_dtype == PKV_F32 ? PKV_F32 : (kv_dtype == PKV_F16 ? PKV_F16 : PKV_BF16);
  if (!pkv::attn_kernel_for(kv_dtype, q_dtype, head_dim, block_size, &k))
    return pkv_fail(PKV_ERR_UNSUPPORTED, "default_num_ctas: no kernel for kv_dtype %d head_dim %d", kv_dtype, head_dim);
  const int n = pkv::resident_ctas(k);
  if (n <= 0) return pkv_fail(PKV_ERR_CUDA, "default_num_ctas: occupancy query failed: %s", cudaGetErrorString(cudaGetLastError()));
  *num_ctas = n;
  return PKV_OK;
}

// Structural check of a host plan: every index the kernels follow stays inside
// the plan and the workspace (lengths are checked against the device arrays by
// the kernels themselves).
// merge_rows receives the most rows of any one merge (the merge grid's y extent in 16-row chunks).
// heads4_ok: the decode-tile kernel of this pool takes four-head items.
static pkv_status validate_plan(const PkvPlanHeader* h, int g, int hkv, int max_rows, bool tc, bool heads4_ok,
                                int* merge_rows) {
  const char* base = reinterpret_cast<const char*>(h);
  const uint64_t bytes = h->bytes;
  if (bytes < sizeof(PkvPlanHeader) + PKV_PLAN_COUNTER_BYTES || (bytes & 255))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan size %llu", (unsigned long long)bytes);
  auto inside = [&](uint64_t off, uint64_t n, uint64_t sz) { return off + n * sz <= bytes - PKV_PLAN_COUNTER_BYTES; };
  if (h->n_items < 0 || h->n_tc_items < 0 || h->n_reduce < 0 || h->n_parts < 0 || h->n_part_rows < 0 ||
      h->total_q < 0 || !inside(h->items_off, h->n_items, sizeof(PkvItem)) ||
      !inside(h->tc_items_off, h->n_tc_items, sizeof(PkvItem)) || !inside(h->reduce_off, h->n_reduce, sizeof(PkvReduce)) ||
      !inside(h->parts_off, h->n_parts, sizeof(int32_t)) || h->num_ctas <= 0 || (h->n_tc_items > 0 && h->tc_num_ctas <= 0))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan sections out of range");
  if (h->n_tc_items > 0 && !tc) return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan has tcgen05 items for a pool without that kernel");
  if ((h->flags & ~(PKV_PLAN_CORUN | PKV_PLAN_HEADS4)) != 0) return pkv_fail(PKV_ERR_PLAN, "paged_attention: unknown plan flags");
  const bool heads4 = (h->flags & PKV_PLAN_HEADS4) != 0;
  if (heads4 && (!heads4_ok || hkv % 4 != 0))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: four-head plan for a pool or head count without that kernel");
  if ((h->flags & PKV_PLAN_CORUN) != 0 && (h->n_items == 0 || h->n_tc_items == 0))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: side-by-side plan without both item lists");
  if (h->n_rows < 0 || !inside(h->rows_off, h->n_rows, sizeof(int32_t)))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan token list out of range");
  const int32_t* rows_list = reinterpret_cast<const int32_t*>(base + h->rows_off);
  auto check_items = [&](uint32_t off, int n, int lo, int hi, bool tc_list, const char* what) -> pkv_status {
    const PkvItem* items = reinterpret_cast<const PkvItem*>(base + off);
    for (int i = 0; i < n; ++i) {
      const PkvItem& it = items[i];
      const int64_t rows = int64_t(it.n_q) * g;
      // Listed query tokens (shared-prefix group tiles, tensor-memory list, partial rows only).
      const bool listed = it.pos0 <= -2;
      const int64_t loff = -2 - int64_t(it.pos0);
      if (listed) {
        if (!tc_list || it.part_row < 0 || loff + it.n_q > h->n_rows)
          return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan %s %d lists bad tokens", what, i);
        for (int k = 0; k < it.n_q; ++k) {
          const int32_t tok = rows_list[loff + k];
          if (tok < 0 || tok >= h->total_q) return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan %s %d lists bad tokens", what, i);
        }
      }
      // A four-head item (decode-tile list of a PKV_PLAN_HEADS4 plan) spans heads kv_head .. + 3
      // and their partial rows.
      const int nh = heads4 && !tc_list ? 4 : 1;
      if (nh == 4 && (rows > PKV_HEADS4_ROWS || it.kv_head % 4 != 0))
        return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan %s %d is not a four-head item", what, i);
      if (it.n_q <= 0 || rows < lo || rows > hi || it.kv_head < 0 || it.kv_head + nh > hkv || it.q_begin < 0 ||
          (!listed && int64_t(it.q_begin) + it.n_q > h->total_q) || it.k_begin < 0 || it.k_begin > it.k_end ||
          it.part_row < -1 || (it.part_row >= 0 && int64_t(it.part_row) + nh * rows > h->n_part_rows))
        return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan %s %d out of range", what, i);
    }
    return PKV_OK;
  };
  if (pkv_status s = check_items(h->items_off, h->n_items, 1, max_rows, false, "item"); s != PKV_OK) return s;
  if (pkv_status s = check_items(h->tc_items_off, h->n_tc_items, PKV_DECODE_ROWS + 1, PKV_TILE_ROWS_TC, true,
                                 "tcgen05 item");
      s != PKV_OK)
    return s;
  const PkvReduce* reds = reinterpret_cast<const PkvReduce*>(base + h->reduce_off);
  const int32_t* parts = reinterpret_cast<const int32_t*>(base + h->parts_off);
  *merge_rows = 0;
  for (int i = 0; i < h->n_reduce; ++i) {
    const PkvReduce& r = reds[i];
    const int64_t rows = int64_t(r.n_q) * g;
    *merge_rows = std::max(*merge_rows, int(std::min<int64_t>(rows, PKV_TILE_ROWS_TC)));
    if (r.n_q <= 0 || rows > PKV_TILE_ROWS_TC || r.kv_head < 0 || r.kv_head >= hkv || r.q_begin < 0 ||
        int64_t(r.q_begin) + r.n_q > h->total_q || r.parts_begin < 0 || r.n_parts < 0 ||
        int64_t(r.parts_begin) + r.n_parts > h->n_parts)
      return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan merge %d out of range", i);
    for (int p = 0; p < r.n_parts; ++p) {
      const int32_t row = parts[r.parts_begin + p];
      if (row < 0 || int64_t(row) + rows > h->n_part_rows)
        return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan merge %d part %d out of range", i, p);
    }
  }
  return PKV_OK;
}

// Under stream capture the record must be external, so that the graph records
// the event each time it runs; outside capture it is a plain record.
static cudaError_t record_event(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                             : cudaEventRecord(ev, st);
}

extern "C" pkv_status pkv_paged_attention_timed(const pkv_cache* cache, const void* q, int32_t q_dtype,
                                                int32_t num_q_heads, const int32_t* cu_q_lens,
                                                const int32_t* seq_lens, const int32_t* block_tables,
                                                int32_t max_blocks, int32_t num_seqs, float softmax_scale,
                                                int32_t causal, const void* plan, void* out, float* out_lse,
                                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                                void* stream, void* kernels_begin, void* kernels_end) {
  if (!cache || !plan) return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: cache and plan are required");
  const pkv_cache& c = *cache;
  const PkvPlanHeader* h = static_cast<const PkvPlanHeader*>(plan);
  if (h->magic != PKV_PLAN_MAGIC) return pkv_fail(PKV_ERR_PLAN, "paged_attention: not a plan buffer");
  if (c.num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % c.num_kv_heads != 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: num_q_heads %d, num_kv_heads %d", num_q_heads, c.num_kv_heads);
  if (!pkv_is_pow2(c.block_size) || c.block_size < 2)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: block_size %d is not a power of two > 1", c.block_size);
  if (c.num_layers <= 0 || c.layer < 0 || c.layer >= c.num_layers || c.num_blocks <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: bad cache shape");
  if (h->num_seqs != num_seqs || h->num_q_heads != num_q_heads || h->num_kv_heads != c.num_kv_heads ||
      h->head_dim != c.head_dim || h->block_size != c.block_size || h->kv_dtype != c.kv_dtype ||
      h->causal != (causal ? 1 : 0) || h->window < 0 || (h->window > 0 && !causal) || h->wait_limit_kcycles < 0 ||
      (h->debug_flags & ~PKV_DEBUG_WITHHOLD_LOADS))
    return pkv_fail(PKV_ERR_PLAN, "paged_attention: plan was made for other shapes");
  pkv::AttnKernel k;
  if (!pkv::attn_kernel_for(c.kv_dtype, q_dtype, c.head_dim, c.block_size, &k))
    return pkv_fail(PKV_ERR_UNSUPPORTED, "paged_attention: kv_dtype %d with q_dtype %d, head_dim %d", c.kv_dtype,
                    q_dtype, c.head_dim);
  if ((c.kv_dtype == PKV_FP8_E4M3 || c.kv_dtype == PKV_NVFP4) && (!c.k_scale || !c.v_scale))
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: fp8 and NVFP4 pools need k_scale and v_scale");
  if (!(softmax_scale > 0.f) || softmax_scale == INFINITY)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: softmax_scale must be positive and finite");
  pkv::AttnKernel ktc{};
  const bool tc = pkv::attn_tc_kernel_for(c.kv_dtype, q_dtype, c.head_dim, c.block_size, &ktc);
  int merge_rows = 0;
  if (pkv_status vs = validate_plan(h, num_q_heads / c.num_kv_heads, c.num_kv_heads, k.max_rows, tc,
                                    pkv_heads4_capable(c.kv_dtype, c.head_dim, c.block_size), &merge_rows);
      vs != PKV_OK)
    return vs;
  const PkvWorkspaceLayout L = pkv_workspace_layout(h->bytes, h->n_part_rows, c.head_dim);
  if (h->n_items == 0 && h->n_tc_items == 0) return PKV_OK;
  if (!workspace || workspace_bytes < L.total)
    return pkv_fail(PKV_ERR_WORKSPACE, "paged_attention: workspace %zu < %llu bytes", workspace_bytes,
                    (unsigned long long)L.total);
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: workspace not 256-byte aligned");
  if (!c.pool || !q || !out || !cu_q_lens || !seq_lens || !block_tables || max_blocks <= 0)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: null pointer or max_blocks <= 0");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(c.pool)) & 15)
    return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention: q, out and pool must be 16-byte aligned");

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  // One copy stages the plan in the workspace and clears the work counters at its end.  A
  // page-locked plan is read by a kernel straight from host memory (launched as a programmatic
  // dependent of whatever precedes it, so it overlaps that work, and finishing only after it);
  // any other plan goes through cudaMemcpyAsync.
  cudaError_t e;
  cudaPointerAttributes pa{};
  const void* plan_dev = nullptr;
  if (cudaPointerGetAttributes(&pa, plan) == cudaSuccess && pa.type == cudaMemoryTypeHost && pa.devicePointer)
    plan_dev = pa.devicePointer;
  else
    cudaGetLastError();  // a failed query leaves no sticky error; take the copy path
  if (plan_dev)
    e = pkv::launch_plan_stage(plan_dev, ws + L.plan_off, h->bytes, st);
  else
    e = cudaMemcpyAsync(ws + L.plan_off, plan, h->bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention: plan upload: %s", cudaGetErrorString(e));
  const int resident = pkv::resident_ctas(k);  // also sets the kernel's shared-memory limit
  const int tc_resident = h->n_tc_items > 0 ? pkv::resident_ctas(ktc) : 1;
  if (resident <= 0 || tc_resident <= 0) return pkv_fail(PKV_ERR_CUDA, "paged_attention: occupancy query failed");
  const char* dplan = ws + L.plan_off;
  pkv::AttnArgs a{};
  a.pool = c.pool;
  a.num_blocks = c.num_blocks;
  a.num_layers = c.num_layers;
  a.layer = c.layer;
  a.hkv = c.num_kv_heads;
  a.log2_block = pkv_log2(c.block_size);
  a.k_scale = c.k_scale;
  a.v_scale = c.v_scale;
  a.q = q;
  a.out = out;
  a.out_lse = out_lse;
  a.cu_q_lens = cu_q_lens;
  a.seq_lens = seq_lens;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks;
  a.num_seqs = num_seqs;
  a.hq = num_q_heads;
  a.g = num_q_heads / c.num_kv_heads;
  a.softmax_scale = softmax_scale;
  a.items = reinterpret_cast<const PkvItem*>(dplan + h->items_off);
  a.row_tokens = reinterpret_cast<const int32_t*>(dplan + h->rows_off);
  a.n_items = h->n_items;
  a.counter = reinterpret_cast<unsigned int*>(ws + L.counter_off);
  a.part_o = reinterpret_cast<float*>(ws + L.part_o_off);
  a.part_lse = reinterpret_cast<float*>(ws + L.part_lse_off);
  a.status = dev_status;
  a.max_rows = k.max_rows;
  a.window = h->window;
  a.debug_flags = h->debug_flags;
  a.wait_limit = h->wait_limit_kcycles > 0 ? 1000ll * h->wait_limit_kcycles : PKV_DEFAULT_WAIT_CYCLES;
  a.total_q = h->total_q;
  a.heads4 = (h->flags & PKV_PLAN_HEADS4) ? 1 : 0;
  if (kernels_begin) {
    e = record_event(static_cast<cudaEvent_t>(kernels_begin), st);
    if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention: event record: %s", cudaGetErrorString(e));
  }
  const bool corun = (h->flags & PKV_PLAN_CORUN) != 0;
  auto launch_reg = [&]() -> pkv_status {
    if (h->n_items == 0) return PKV_OK;
    const int grid = std::max(1, std::min(std::min(resident, h->num_ctas), h->n_items));
    pkv::AttnArgs r = a;
    r.pdl_role = corun ? 1 : 0;  // side by side: launched beside the tcgen05 kernel
    const cudaError_t le = k.launch(r, grid, st);
    if (le != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention: launch failed: %s", cudaGetErrorString(le));
    return PKV_OK;
  };
  auto launch_tc = [&]() -> pkv_status {
    if (h->n_tc_items == 0) return PKV_OK;
    pkv::AttnArgs t = a;
    t.items = reinterpret_cast<const PkvItem*>(dplan + h->tc_items_off);
    t.n_items = h->n_tc_items;
    t.counter = a.counter + 32;  // 128 bytes on
    t.max_rows = ktc.max_rows;
    t.pdl_role = corun ? 0 : 1;
    const int grid = std::max(1, std::min(std::min(tc_resident, h->tc_num_ctas), h->n_tc_items));
    const cudaError_t le = ktc.launch(t, grid, st);
    if (le != cudaSuccess)
      return pkv_fail(PKV_ERR_CUDA, "paged_attention: tcgen05 launch failed: %s", cudaGetErrorString(le));
    return PKV_OK;
  };
  // Side by side: the tcgen05 tiles first on their share of the SMs, the decode tiles beside
  // them.  Otherwise the decode tiles first and the tcgen05 tiles behind them (its CTAs take the
  // SMs the decode-tile kernel frees as it drains).
  if (corun) {
    if (pkv_status ls = launch_tc(); ls != PKV_OK) return ls;
    if (pkv_status ls = launch_reg(); ls != PKV_OK) return ls;
  } else {
    if (pkv_status ls = launch_reg(); ls != PKV_OK) return ls;
    if (pkv_status ls = launch_tc(); ls != PKV_OK) return ls;
  }
  if (kernels_end) {
    e = record_event(static_cast<cudaEvent_t>(kernels_end), st);
    if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention: event record: %s", cudaGetErrorString(e));
  }
  if (h->n_reduce > 0) {
    pkv::ReduceArgs r{};
    r.reduces = reinterpret_cast<const PkvReduce*>(dplan + h->reduce_off);
    r.parts = reinterpret_cast<const int32_t*>(dplan + h->parts_off);
    r.n_reduce = h->n_reduce;
    r.part_o = a.part_o;
    r.part_lse = a.part_lse;
    r.out = out;
    r.out_lse = out_lse;
    r.out_dtype = q_dtype;
    r.hq = num_q_heads;
    r.g = a.g;
    r.head_dim = c.head_dim;
    e = pkv::launch_plan_reduce(r, merge_rows, st);
    if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention: merge launch failed: %s", cudaGetErrorString(e));
  }
  return PKV_OK;
}

extern "C" pkv_status pkv_paged_attention(const pkv_cache* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                                          const int32_t* cu_q_lens, const int32_t* seq_lens,
                                          const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                          float softmax_scale, int32_t causal, const void* plan, void* out,
                                          float* out_lse, void* workspace, size_t workspace_bytes,
                                          int32_t* dev_status, void* stream) {
  return pkv_paged_attention_timed(cache, q, q_dtype, num_q_heads, cu_q_lens, seq_lens, block_tables, max_blocks,
                                   num_seqs, softmax_scale, causal, plan, out, out_lse, workspace, workspace_bytes,
                                   dev_status, stream, nullptr, nullptr);
}
