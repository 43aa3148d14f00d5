// Routing without any device allocation by the caller.
//
// h3attn_route needs scratch memory for the pooled Q and K centroids, which
// the caller normally provides as a workspace it allocated.  Some callers
// cannot allocate device memory at the moment they route: a host framework
// that owns every byte of device memory through its own pool and forbids
// other allocators, a latency-critical loop where cudaMalloc's implicit
// device synchronisation is unacceptable, or a plugin host that grants a
// fixed memory budget up front.  h3attn_route_static serves them: its scratch
// is a file-scope __device__ array of fixed size that every GPU loading this
// library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "h3attn.h"
#include "kernels.cuh"


namespace {

// 32 MiB of routing scratch (two-part pooled centroids and the score matrix).
constexpr size_t kStaticPooledFloats = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_pooled_scratch[kStaticPooledFloats];

std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_pooled_scratch on the current device (the host-side
// name is only a stand-in and must never reach a kernel).  Looked up once per
// device, on the first call made with that device current.
float* scratch_for_current_device(int* status) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = H3ATTN_ECUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    float* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_pooled_scratch) != cudaSuccess || ptr == nullptr) {
      *status = H3ATTN_ECUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *status = H3ATTN_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int h3attn_route_static(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, int32_t* kv_sel,
                                   void* stream) {
  if (h3attn_workspace_bytes(plan) == 0) return H3ATTN_EINVAL;  // rejects a malformed plan
  if (q == nullptr || k == nullptr || kv_sel == nullptr || plan->n_video_blocks == 0) return H3ATTN_EINVAL;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(k) & 15u) ||
      (reinterpret_cast<uintptr_t>(kv_sel) & 3u))
    return H3ATTN_EALIGN;
  const h3::RouteScratch need = h3::route_scratch_layout(plan->H, plan->d, plan->n_video_blocks);
  if (need.total > kStaticPooledFloats * sizeof(float)) return H3ATTN_EWORKSPACE;
  if (h3::route_smem_bytes(plan->d, plan->n_video_blocks) > (size_t)227 * 1024) return H3ATTN_EUNSUPPORTED;
  int status = H3ATTN_OK;
  float* scratch = scratch_for_current_device(&status);
  if (scratch == nullptr) return status;
  if (h3::launch_route_pipeline(q, k, kv_sel, plan->H, plan->S, plan->d, plan->first_video_block,
                                plan->n_video_blocks, plan->k, scratch, nullptr,
                                static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}
