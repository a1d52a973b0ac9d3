// pod_attn_run_static: the same hybrid-batch attention as pod_attn_run, for
// callers that cannot allocate device memory themselves.
//
// pod_attn_run needs a caller-provided workspace (ticket and queue counters,
// the plan's work tables, split-KV partial results).  Some callers have no way
// to provide one: a plugin hosted inside an inference engine that has reserved
// (almost) all of HBM for its own pools and offers no workspace hook, or a
// latency-critical caller that cannot afford cudaMalloc's implicit device
// synchronisation.  For them this file keeps the workspace in a fixed-size
// device array that lives as long as the library is loaded in the process (on
// every GPU that loads the library).  Nothing here calls cudaMalloc, cudaFree
// or any allocating routine.
#include <cuda_runtime.h>

#include "pod_plan.h"

namespace {

// The workspace shared by every pod_attn_run_static call on a device.
static __device__ __align__(256) unsigned char g_pod_static_scratch[POD_STATIC_SCRATCH_BYTES];

// Device address of the scratch array in the current context.  In host code
// the array's name is only a host-side stand-in, so the kernels must receive
// this address, never the name.  It is looked up on every call rather than
// cached: after cudaDeviceReset (or in another context on the same device) the
// module is loaded again and the array may sit elsewhere, and a cached address
// would then point at unmapped memory.  Once the module is loaded in the
// context the lookup is a table read, not a stream operation.
int scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_pod_static_scratch);
  if (e != cudaSuccess || !p) return POD_ERR_CUDA;
  *out = p;
  return POD_OK;
}

}  // namespace

extern "C" int pod_attn_run_static(const pod_attn_plan_t* plan, const void* q_prefill, const void* q_decode,
                                   const void* k_cache, const void* v_cache, int64_t num_blocks,
                                   const int32_t* block_table, int32_t block_table_stride, const int32_t* kv_lens,
                                   float scale, void* o_prefill, void* o_decode, void* stream) {
  if (!plan) return POD_ERR_INVALID_ARG;
  if (plan->ws_bytes > (int64_t)POD_STATIC_SCRATCH_BYTES) return POD_ERR_WORKSPACE;
  void* ws = nullptr;
  int rc = scratch_address(&ws);
  if (rc != POD_OK) return rc;
  // The array keeps whatever the previous call left in it: re-copy this plan's
  // tables and zero the counters (pod_attn_upload does both) before the run.
  rc = pod_attn_upload(plan, ws, POD_STATIC_SCRATCH_BYTES, stream);
  if (rc != POD_OK) return rc;
  return pod_attn_run(plan, q_prefill, q_decode, k_cache, v_cache, num_blocks, block_table, block_table_stride,
                      kv_lens, scale, o_prefill, o_decode, ws, POD_STATIC_SCRATCH_BYTES, nullptr, stream);
}
