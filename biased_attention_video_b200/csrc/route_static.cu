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
// library holds until the process exits.  The array's first 256 bytes hold
// the status word of these calls (a bounded device-side wait that gave up),
// which h3attn_route_static_check reports and clears.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "h3attn.h"
#include "kernels.cuh"


namespace {

// 64 MiB: a 256-byte status header, then the routing scratch (the three-part
// bf16 pooled centroids and the score matrix).
constexpr size_t kStaticBytes = size_t(64) << 20;
constexpr size_t kStatusHeader = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_pooled_scratch[kStaticBytes / sizeof(float)];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DeviceEntry {
  unsigned long long ctx_id;  // context the address was looked up in
  uint8_t* base;              // device address of g_pooled_scratch in that context
};

std::mutex g_setup_mutex;
DeviceEntry g_entries[kMaxDevices] = {};

template <typename Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

// Device address of g_pooled_scratch in the current context (the host-side
// name is only a stand-in and must never reach a kernel).  Looked up on the
// first call made with a device current, and again whenever that device's
// current context is a different one (after cudaDeviceReset the module is
// loaded again, at a new address): the cache is keyed on the context's
// process-unique id.
uint8_t* static_base(int* status) {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  *status = H3ATTN_ECUDA;
  int dev = -1;
  if (get_current == nullptr || get_id == nullptr) return nullptr;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return nullptr;
  if (ctx == nullptr) {  // runtime not initialised on this thread yet: make the primary context current
    if (cudaSetDevice(dev) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceEntry& e = g_entries[dev];
  if (e.base == nullptr || e.ctx_id != id) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_pooled_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    e.base = static_cast<uint8_t*>(ptr);
    e.ctx_id = id;
  }
  *status = H3ATTN_OK;
  return e.base;
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
  if (need.total > kStaticBytes - kStatusHeader) return H3ATTN_EWORKSPACE;
  if (h3::route_smem_bytes(plan->d, plan->n_video_blocks) > (size_t)h3::kMaxSmem) return H3ATTN_EUNSUPPORTED;
  int status = H3ATTN_OK;
  uint8_t* base = static_base(&status);
  if (base == nullptr) return status;
  if (h3::launch_route_pipeline(q, k, kv_sel, plan->H, plan->S, plan->d, plan->first_video_block,
                                plan->n_video_blocks, plan->k, base + kStatusHeader, reinterpret_cast<int*>(base),
                                static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

extern "C" int h3attn_route_static_check(void* stream) {
  int rc = H3ATTN_OK;
  uint8_t* base = static_base(&rc);
  if (base == nullptr) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return H3ATTN_ECUDA;
  int status = 0;
  if (cudaMemcpy(&status, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return H3ATTN_ECUDA;
  if (status != 0 && cudaMemset(base, 0, sizeof(int)) != cudaSuccess) return H3ATTN_ECUDA;
  if (status == h3::kStatusTimeout) return H3ATTN_ETIMEOUT;
  if (status == h3::kStatusData) return H3ATTN_EDATA;
  return status == 0 ? H3ATTN_OK : H3ATTN_ECUDA;
}
