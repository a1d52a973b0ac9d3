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

#include <mutex>

#include "pod_plan.h"

namespace {

// The workspace shared by every pod_attn_run_static call on a device.
static __device__ __align__(256) unsigned char g_pod_static_scratch[POD_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in, so
// the kernels must receive this address, never the name.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return POD_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return POD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pod_static_scratch);
    if (e != cudaSuccess || !p) return POD_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
