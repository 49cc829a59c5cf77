// wf_chunk_causal_attn_noalloc: the attention entry point for callers that
// cannot allocate device memory.
//
// The only scratch the attention kernels use is their workspace status block.
// Here it lives in a file-scope device array that the library reserves on
// every GPU it is loaded on, for the life of the process, so the caller passes
// only inputs and outputs.  In host code the array's name is a host-side
// stand-in, not a device address: its device address is fetched once per
// device with cudaGetSymbolAddress (with that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "wf.h"
#include "wf_plan.h"

namespace {

constexpr size_t kStaticScratchBytes = 4096;  // stated maximum of the static scratch
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the static scratch on the current device (set-up on the
// first call per device).  Returns nullptr if the runtime call fails.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_attn_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" wf_status wf_chunk_causal_attn_noalloc(const void* host_plan, const void* dev_plan, const void* q_rot,
                                                  const void* k_pool, const void* v_pool, void* out, float* lse,
                                                  float softmax_scale, wf_stream_t stream) {
  if (!host_plan) return WF_ERR_INVALID_ARG;
  const size_t need = wf_attn_workspace_bytes(host_plan);
  if (need == 0) return WF_ERR_PLAN;
  if (need > kStaticScratchBytes) return WF_ERR_CAPACITY;
  void* scratch = scratch_on_current_device();
  if (!scratch) return WF_ERR_CUDA;
  // the kernels only ever set the status word; each call starts from zero
  if (cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return WF_ERR_CUDA;
  }
  return wf_chunk_causal_attn(host_plan, dev_plan, q_rot, k_pool, v_pool, out, lse, softmax_scale, scratch, need,
                              stream);
}

extern "C" wf_status wf_attn_noalloc_status(wf_stream_t stream, int32_t* detail) {
  void* scratch = scratch_on_current_device();
  if (!scratch) return WF_ERR_CUDA;
  return wf_attn_workspace_status(scratch, stream, detail);
}
