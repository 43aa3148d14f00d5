// Block mean-pool of Q and K ("H3 SLA Attention", "How it works": each block
// is represented by its pooled centroid), the per-key-block descriptors used
// by the attention kernel, and the bounded-wait self-test.
#include <cuda_runtime.h>
#include <cstdint>

#include "fastmath.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per (tensor, head, block): 64 rows x D bf16, read as 16-byte
// vectors (D/8 lanes per row, 256/D rows per pass), summed in fp32, scaled by
// 1 / valid rows.  Memory-bound: every input byte is read exactly once.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ x0, float* __restrict__ out0,
                                                   const uint16_t* __restrict__ x1, float* __restrict__ out1,
                                                   int H, int S, int first_block, int n_out) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  const long long warp_id = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long per_tensor = (long long)H * n_out;
  const int n_tensors = x1 != nullptr ? 2 : 1;
  if (warp_id >= per_tensor * n_tensors) return;
  const int t = (int)(warp_id / per_tensor);
  const long long rem = warp_id % per_tensor;
  const int h = (int)(rem / n_out);
  const int ob = (int)(rem % n_out);
  const int b = first_block + ob;
  const uint16_t* x = t == 0 ? x0 : x1;
  float* out = t == 0 ? out0 : out1;
  const int row0 = b * kBlock;
  const int nrows = min(kBlock, S - row0);
  const int chunk = lane % kLanesPerRow;
  const int rsub = lane / kLanesPerRow;
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)h * S + row0) * D) + chunk;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  constexpr int kPasses = kBlock / kRowsPerPass;
  if (nrows == kBlock) {
    constexpr int kBatch = 8;  // 16-byte loads in flight per lane
#pragma unroll
    for (int i0 = 0; i0 < kPasses; i0 += kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        v[i] = __ldg(src + (size_t)((i0 + i) * kRowsPerPass + rsub) * kLanesPerRow);
#pragma unroll
      for (int i = 0; i < kBatch; ++i) add_bf16x8(acc, v[i]);
    }
  } else {
    for (int r = rsub; r < nrows; r += kRowsPerPass) add_bf16x8(acc, __ldg(src + (size_t)r * kLanesPerRow));
  }
#pragma unroll
  for (int o = kLanesPerRow; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
  if (rsub == 0) {
    const float inv = 1.0f / (float)nrows;
    float4* dst = reinterpret_cast<float4*>(out + ((size_t)h * n_out + ob) * D + chunk * 8);
    dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

// kv_desc[b].x = valid rows | kind << 8 with kind 0: no guide row, 1: every
// row is a guide row and all share one time (stored in .y), 2: anything else
// holding guide rows (penalty evaluated per key).
__global__ void kv_desc_kernel(const uint8_t* __restrict__ seg, const float* __restrict__ times, int S,
                               int n_blocks, uint4* __restrict__ desc, float* __restrict__ gtime,
                               uint32_t* __restrict__ slow_bits) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;  // 32 consecutive blocks per warp
  bool slow = false;
  if (b < n_blocks) {
    const int lo = b * kBlock;
    const int n = min(kBlock, S - lo);
    const float nan = __int_as_float(0x7FC00000);
    // each row's key time: its time if it is a guide row, NaN otherwise; the
    // block splits into at most two runs of equal key time (NaN == NaN here)
    bool any_guide = false, two_runs = true;
    int split = n;
    uint32_t ta = 0u, tb = 0u;
    for (int r = 0; r < kBlock; ++r) {
      const bool guide = r < n && seg[lo + r] == kSegGuide;
      const float t = guide ? (times != nullptr ? times[lo + r] : 0.0f) : nan;
      if (gtime != nullptr && times != nullptr) gtime[lo + r] = t;
      if (r >= n) continue;
      any_guide |= guide;
      const uint32_t tbits = __float_as_uint(t);
      if (r == 0) {
        ta = tb = tbits;
      } else if (split == n) {
        if (tbits != ta) {
          split = r;
          tb = tbits;
        }
      } else if (tbits != tb) {
        two_runs = false;
      }
    }
    const uint32_t kind = !any_guide ? 0u : (two_runs ? 1u : 2u);
    desc[b] = make_uint4((uint32_t)n | (kind << 8) | ((uint32_t)split << 16), ta, tb, 0u);
    // (penalty off -- times null -- leaves only the validity test)
    slow = n < kBlock || (times != nullptr && (kind == 2u || (kind == 1u && split < n && (split & 15) != 0)));
  }
  const uint32_t word = __ballot_sync(0xFFFFFFFFu, slow);
  if ((threadIdx.x & 31) == 0 && b < ((n_blocks + 31) & ~31)) slow_bits[b >> 5] = word;
}

__global__ void selftest_timeout_kernel(int* status, uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives
    fence_mbar_init();
    bool done = false;
    for (uint32_t i = 0; i < polls && !done; ++i) done = mbar_try_wait(&bar, 0);
    if (!done) atomicCAS(status, 0, kStatusTimeout);
  }
}

}  // namespace


cudaError_t launch_pool(const uint16_t* x0, float* out0, const uint16_t* x1, float* out1, int H, int S, int d,
                        int first_block, int n_out, cudaStream_t stream) {
  const long long warps = (long long)H * n_out * (x1 != nullptr ? 2 : 1);
  const unsigned grid = (unsigned)((warps + 7) / 8);
  if (grid == 0) return cudaSuccess;
  if (d == 64)
    pool_kernel<64><<<grid, 256, 0, stream>>>(x0, out0, x1, out1, H, S, first_block, n_out);
  else
    pool_kernel<128><<<grid, 256, 0, stream>>>(x0, out0, x1, out1, H, S, first_block, n_out);
  return cudaGetLastError();
}

cudaError_t launch_kv_desc(const uint8_t* seg, const float* times, int S, int n_blocks, uint4* kv_desc,
                           float* gtime, uint32_t* slow, cudaStream_t stream) {
  kv_desc_kernel<<<(n_blocks + 127) / 128, 128, 0, stream>>>(seg, times, S, n_blocks, kv_desc, gtime, slow);
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(int* status, uint32_t polls, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(status, polls);
  return cudaGetLastError();
}

}  // namespace h3
