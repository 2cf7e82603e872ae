// Launch arguments of the attention and merge kernels (host and device).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan_format.h"

namespace pkv {

struct AttnArgs {
  const void* pool;
  int64_t num_blocks;
  int32_t num_layers, layer, hkv, log2_block;
  const float* k_scale;  // fp8 pools only
  const float* v_scale;
  const void* q;
  void* out;
  float* out_lse;
  const int32_t* cu_q_lens;
  const int32_t* seq_lens;
  const int32_t* block_tables;
  int32_t max_blocks, num_seqs, hq, g;
  float softmax_scale;
  const PkvItem* items;  // device copy of the plan's items
  const int32_t* row_tokens;  // device copy of the plan's listed query tokens (group tiles)
  int32_t n_items;
  unsigned int* counter;  // work counter, zeroed before the launch
  float* part_o;          // [n_part_rows][head_dim]
  float* part_lse;        // [n_part_rows]
  int32_t* status;
  int32_t max_rows;       // rows per item this kernel accepts
  int32_t window;         // limited attention window (causal rows see keys pos - window < t <= pos); 0 = none
  int32_t debug_flags;    // PKV_DEBUG_* from the plan (0 in normal use)
  long long wait_limit;   // SM cycles every pipeline wait may take before it gives up
  int32_t total_q;        // query tokens of the batch (rows of q / Hq)
  // Place among the attention kernels launched as programmatic dependents: 0 = first (waits for
  // the work ahead at its start, then lets the next kernel launch), 1 = second (launched beside
  // the first, which waited for the work ahead before letting it launch; it waits for the first
  // before it finishes, so the merge after it sees both).
  int32_t pdl_role;
  // 1: the plan's decode-tile items each cover four KV heads, kv_head .. kv_head + 3
  // (PKV_PLAN_HEADS4); consumer warp w runs head kv_head + w.
  int32_t heads4;
};

struct ReduceArgs {
  const PkvReduce* reduces;
  const int32_t* parts;
  int32_t n_reduce;
  const float* part_o;
  const float* part_lse;
  void* out;
  float* out_lse;
  int32_t out_dtype, hq, g, head_dim;
};

// Kernel selection for one (pool dtype, q dtype, head_dim).
struct AttnKernel {
  const void* fn;
  int threads;
  int smem;
  cudaError_t (*launch)(const AttnArgs&, int grid, cudaStream_t);
  int max_rows;  // rows per item the kernel accepts
  // The variant for four-head plans (same threads and shared memory), launched by `launch`
  // when AttnArgs::heads4 is set; null where there is none.
  const void* fn_heads4 = nullptr;
};
// Picks the TMA kernel where it applies (block size >= 8, 128/256-byte rows),
// else the cp.async tensor-core kernel, and the CUDA-core kernel for fp32 pools.
bool attn_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k);
bool attn_tma_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k);
// tcgen05 kernel for the tiles of more than 16 rows of a 16-bit pool or of an fp8 pool of
// head_dim 128 (attn_tc.cu).
bool attn_tc_kernel_for(int kv_dtype, int q_dtype, int head_dim, int block_size, AttnKernel* k);
// SM count x occupancy of a kernel on the current device (cached per device).
int resident_ctas(const AttnKernel& k);
// The pool as a 5-D TMA tensor (attn_tma.cu): head_dim, slot, kv head, 2*layer + K|V, block;
// boxes of 128 bytes x box_rows slots x 1 head x box_kv x 1 block, 128-byte swizzle.
bool make_pool_map(const AttnArgs& a, int head_dim, int elem, CUtensorMapDataType dt, int box_rows, int box_kv,
                   CUtensorMap* map);
// The plan's merges (reduce.cu); max_rows = the most rows of any one merge, which sizes the
// grid's y dimension in chunks of 16 rows.
cudaError_t launch_plan_reduce(const ReduceArgs& r, int max_rows, cudaStream_t st);
// Copy `bytes` (a multiple of 16) of a page-locked host plan, addressed through its device
// alias, into the workspace (reduce.cu).  Launched as a programmatic dependent; the grid
// completes only after the work ahead of it on the stream.
cudaError_t launch_plan_stage(const void* plan_dev, void* dst, uint64_t bytes, cudaStream_t st);

// Launch `kernel` with programmatic stream serialization: it may begin while the
// kernel ahead of it on the stream is still running (and must call pdl_wait
// before it depends on that kernel's results).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace pkv
