// paged_attention without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run
// attention: a plug-in that receives only the input and output pointers from a
// host framework, an allocator-free inference runtime, or code running where a
// cudaMalloc would synchronise the device or break a memory budget fixed ahead
// of time.  For them this file keeps the attention launch's scratch (the plan
// copy, the work counter and the split-KV partial states) in one statically
// sized device array that the library carries with it.
//
// Rules of this entry point:
//   * The array holds PKV_NOALLOC_SCRATCH_BYTES (32 MiB) on every GPU that loads
//     the library, for the life of the process.  A plan whose workspace exceeds
//     it is rejected with PKV_ERR_WORKSPACE (plan with fewer splits, or use
//     pkv_paged_attention with a workspace of your own).
//   * The first call on a device looks up the array's device address on that
//     device (cudaGetSymbolAddress, with that device current).  Make that first
//     call outside any stream capture.  The address is kept per device together
//     with the identity of the device's current CUDA context; when the context
//     changes (cudaDeviceReset, or a context destroyed and made again) the
//     module is loaded anew and the array may move, so the next call looks the
//     address up again -- that call, too, must be made outside stream capture.
//   * Every call on a device uses the same array, and the array keeps whatever
//     the last call left there.  The work counters are cleared by each call's plan
//     upload; partial states are fully written before they are read.
//     Calls whose work overlaps on the GPU (other streams, other host threads
//     without ordering) race on the array: order them on one stream.
//   * Nothing here allocates or frees memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "plan_format.h"

#define PKV_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char pkv_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_setup_mutex;
void* g_scratch_ptr[PKV_NOALLOC_MAX_DEVICES] = {};
unsigned long long g_scratch_ctx[PKV_NOALLOC_MAX_DEVICES] = {};  // context the address belongs to

// Identity of the calling thread's current CUDA context (0 if the driver cannot say): the
// driver's unique context id, reached through the runtime's driver entry points.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

// Device address of the scratch array on the current device, looked up on the first call per
// device and again whenever that device's context has changed since.
pkv_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pkv_fail(PKV_ERR_CUDA, "paged_attention_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= PKV_NOALLOC_MAX_DEVICES)
    return pkv_fail(PKV_ERR_UNSUPPORTED, "paged_attention_noalloc: device %d beyond %d", dev, PKV_NOALLOC_MAX_DEVICES);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  const unsigned long long ctx = g_scratch_ptr[dev] ? current_context_id() : 0;
  if (!g_scratch_ptr[dev] || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, pkv_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return pkv_fail(PKV_ERR_CUDA, "paged_attention_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the symbol lookup made the context current if needed
  }
  *out = g_scratch_ptr[dev];
  return PKV_OK;
}
}  // namespace

extern "C" pkv_status pkv_paged_attention_noalloc(const pkv_cache* cache, const void* q, int32_t q_dtype,
                                                  int32_t num_q_heads, const int32_t* cu_q_lens,
                                                  const int32_t* seq_lens, const int32_t* block_tables,
                                                  int32_t max_blocks, int32_t num_seqs, float softmax_scale,
                                                  int32_t causal, const void* plan, void* out, float* out_lse,
                                                  int32_t* dev_status, void* stream) {
  if (!cache || !plan) return pkv_fail(PKV_ERR_INVALID_ARG, "paged_attention_noalloc: cache and plan are required");
  const PkvPlanHeader* h = static_cast<const PkvPlanHeader*>(plan);
  if (h->magic != PKV_PLAN_MAGIC) return pkv_fail(PKV_ERR_PLAN, "paged_attention_noalloc: not a plan buffer");
  if (h->n_part_rows < 0 || cache->head_dim <= 0)
    return pkv_fail(PKV_ERR_PLAN, "paged_attention_noalloc: bad plan or head_dim");
  const uint64_t need = pkv_workspace_layout(h->bytes, h->n_part_rows, cache->head_dim).total;
  if (need > PKV_NOALLOC_SCRATCH_BYTES)
    return pkv_fail(PKV_ERR_WORKSPACE,
                    "paged_attention_noalloc: this plan needs %llu bytes of scratch, more than the built-in %llu; "
                    "plan with fewer key splits or call pkv_paged_attention with your own workspace",
                    (unsigned long long)need, (unsigned long long)PKV_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  pkv_status st = scratch_for_current_device(&scratch);
  if (st != PKV_OK) return st;
  return pkv_paged_attention(cache, q, q_dtype, num_q_heads, cu_q_lens, seq_lens, block_tables, max_blocks, num_seqs,
                             softmax_scale, causal, plan, out, out_lse, scratch, PKV_NOALLOC_SCRATCH_BYTES, dev_status,
                             stream);
}
