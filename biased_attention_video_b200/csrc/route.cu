// Pooled-score routing ("H3 SLA Attention", "How it works": every query block
// is scored against every key block with one small pooled matmul and only the
// top 1 - sparsity_ratio fraction is kept).
//
// One CTA scores kQB video query blocks of one head against all video key
// blocks (fp32 dot products of the pooled centroids, kept in shared memory),
// then each warp selects the k best of a row by a 4-pass radix select on the
// order-preserving integer image of the fp32 score, ties to the lower block,
// and writes the chosen blocks in ascending order.  The 1/sqrt(d) scale is a
// positive constant and does not change the order, so it is not applied.
#include <cuda_runtime.h>
#include <cstdint>

#include "kernels.cuh"

namespace h3 {
namespace {

constexpr int kQB = 16;      // query blocks per CTA
constexpr int kKC = 64;      // key blocks per shared-memory chunk
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D>
__global__ void __launch_bounds__(kThreads) route_kernel(const float* __restrict__ qp, const float* __restrict__ kp,
                                                         int32_t* __restrict__ sel, int n_video, int k,
                                                         int first_video_block) {
  constexpr int kPad = D + 4;  // float4-aligned row pitch, conflict-free 16-byte reads
  extern __shared__ float4 smem4[];
  float* qs = reinterpret_cast<float*>(smem4);           // [kQB][kPad]
  float* ks = qs + kQB * kPad;                           // [kKC][kPad]
  float* scores = ks + kKC * kPad;                       // [kQB][n_video]
  uint32_t* hist = reinterpret_cast<uint32_t*>(scores + kQB * n_video);  // [8 warps][256]

  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kQB;
  const int nq = min(kQB, n_video - i0);
  const int tid = threadIdx.x;
  const float* qph = qp + (size_t)h * n_video * D;
  const float* kph = kp + (size_t)h * n_video * D;

  for (int idx = tid; idx < kQB * (D / 4); idx += kThreads) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nq) v = reinterpret_cast<const float4*>(qph + (size_t)(i0 + r) * D)[c4];
    reinterpret_cast<float4*>(qs + r * kPad)[c4] = v;
  }

  // ---- scores: thread (ty, tx) computes query block ty x key blocks tx + 16 e, e < 4
  const int ty = tid >> 4, tx = tid & 15;
  for (int j0 = 0; j0 < n_video; j0 += kKC) {
    __syncthreads();
    const int nk = min(kKC, n_video - j0);
    for (int idx = tid; idx < kKC * (D / 4); idx += kThreads) {
      const int r = idx / (D / 4), c4 = idx % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nk) v = reinterpret_cast<const float4*>(kph + (size_t)(j0 + r) * D)[c4];
      reinterpret_cast<float4*>(ks + r * kPad)[c4] = v;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float4* qrow = reinterpret_cast<const float4*>(qs + ty * kPad);
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 a = qrow[c4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 b = reinterpret_cast<const float4*>(ks + (tx + 16 * e) * kPad)[c4];
        acc[e] = fmaf(a.x, b.x, acc[e]);
        acc[e] = fmaf(a.y, b.y, acc[e]);
        acc[e] = fmaf(a.z, b.z, acc[e]);
        acc[e] = fmaf(a.w, b.w, acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = tx + 16 * e;
      if (ty < nq && j < nk) scores[ty * n_video + j0 + j] = acc[e];
    }
  }
  __syncthreads();

  // ---- top-k per row: radix select of the k-th largest key, then an ordered sweep
  const int warp = tid >> 5, lane = tid & 31;
  uint32_t* wh = hist + warp * 256;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int row = warp; row < nq; row += kThreads / 32) {
    const float* s = scores + row * n_video;
    uint32_t prefix = 0, pmask = 0;
    int need = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) wh[lane * 8 + i] = 0;
      __syncwarp();
      for (int j = lane; j < n_video; j += 32) {
        const uint32_t key = order_key(s[j]);
        if ((key & pmask) == prefix) atomicAdd(wh + ((key >> shift) & 255u), 1u);
      }
      __syncwarp();
      // lane l holds digits 255-8l .. 248-8l (descending)
      uint32_t c[8];
      uint32_t sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = wh[255 - 8 * lane - e];
        sum += c[e];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      const bool here = excl < (uint32_t)need && (uint32_t)need <= incl;
      const uint32_t who = __ballot_sync(0xFFFFFFFFu, here);
      const int src = __ffs(who) - 1;
      uint32_t digit = 0, greater = 0;
      if (here) {
        uint32_t cum = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + c[e] >= (uint32_t)need) {
            digit = 255u - 8u * lane - e;
            greater = cum;
            break;
          }
          cum += c[e];
        }
      }
      digit = __shfl_sync(0xFFFFFFFFu, digit, src);
      greater = __shfl_sync(0xFFFFFFFFu, greater, src);
      need -= (int)greater;
      prefix |= digit << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    // keys > prefix are taken; `need` keys == prefix, the lowest blocks first
    int32_t* dst = sel + ((size_t)blockIdx.y * n_video + i0 + row) * k;
    int pos = 0, eq_seen = 0;
    for (int jb = 0; jb < n_video; jb += 32) {
      const int j = jb + lane;
      const uint32_t key = j < n_video ? order_key(s[j]) : 0u;
      const bool gt = j < n_video && key > prefix;
      const bool eq = j < n_video && key == prefix;
      const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, eq);
      const bool take = gt || (eq && eq_seen + __popc(eqm & lt_mask) < need);
      const uint32_t tm = __ballot_sync(0xFFFFFFFFu, take);
      const int slot = pos + __popc(tm & lt_mask);
      if (take && slot < k) dst[slot] = first_video_block + j;
      pos += __popc(tm);
      eq_seen += __popc(eqm);
    }
  }
}

}  // namespace

cudaError_t launch_route(const float* qp, const float* kp, int32_t* kv_sel, int H, int d, int n_video, int k,
                         int first_video_block, cudaStream_t stream) {
  const int pad = d + 4;
  const size_t smem = sizeof(float) * ((size_t)kQB * pad + (size_t)kKC * pad + (size_t)kQB * n_video) +
                      sizeof(uint32_t) * 8 * 256;
  dim3 grid((n_video + kQB - 1) / kQB, H);
  if (d == 64) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_kernel<64><<<grid, kThreads, smem, stream>>>(qp, kp, kv_sel, n_video, k, first_video_block);
  } else {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_kernel<128><<<grid, kThreads, smem, stream>>>(qp, kp, kv_sel, n_video, k, first_video_block);
  }
  return cudaGetLastError();
}

size_t route_smem_bytes(int d, int n_video) {
  return sizeof(float) * ((size_t)kQB * (d + 4) + (size_t)kKC * (d + 4) + (size_t)kQB * n_video) +
         sizeof(uint32_t) * 8 * 256;
}

}  // namespace h3
