// Per-token int8 quantisation of Q and K for the int8-QK attention path
// ("H3 SLA Attention", inputs table, use_int8_qk: Q and K quantised to int8
// per token with a dynamic scale before the QK dot product; PV unchanged).
//
// Per row x of d values: a = max|x|, scale s = a / 127, codes
// clamp(rint(x * (127 / a)), -127, 127), all in fp32 with round-to-nearest-even
// (IEEE quotients and product, conversion ties to even); a row of zeros gets
// s = 0 and zero codes.  Scales are stored per head with a padded stride of
// whole 64-row blocks; padding rows get s = 0.
//
// HBM-bound: one warp per row, d / 32 consecutive elements per lane.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace h3 {
namespace {

template <int D>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                         int8_t* __restrict__ q8, int8_t* __restrict__ k8,
                                                         float* __restrict__ sq, float* __restrict__ sk, int H, int S,
                                                         int stride) {
  constexpr int kPer = D / 32;  // elements per lane: 4 (d = 128) or 2 (d = 64)
  const long long warp_id = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long per_tensor = (long long)H * stride;
  if (warp_id >= 2 * per_tensor) return;  // warp-uniform
  const bool is_k = warp_id >= per_tensor;
  const long long rem = is_k ? warp_id - per_tensor : warp_id;
  const int h = (int)(rem / stride), r = (int)(rem % stride);
  float* scale = (is_k ? sk : sq) + (size_t)h * stride + r;
  if (r >= S) {
    if (lane == 0) *scale = 0.0f;
    return;
  }
  const size_t off = ((size_t)h * S + r) * D + (size_t)lane * kPer;
  const uint16_t* src = (is_k ? k : q) + off;
  float v[kPer];
  if constexpr (kPer == 4) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(src));
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xFFFF0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(src));
    v[0] = __uint_as_float(w << 16);
    v[1] = __uint_as_float(w & 0xFFFF0000u);
  }
  // |x| of finite floats orders like its bit pattern
  uint32_t amax = 0u;
#pragma unroll
  for (int i = 0; i < kPer; ++i) amax = max(amax, __float_as_uint(v[i]) & 0x7FFFFFFFu);
  const float a = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, amax));
  uint32_t packed = 0u;
  if (a > 0.0f) {
    const float inv = __fdiv_rn(127.0f, a);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = min(127, max(-127, __float2int_rn(__fmul_rn(v[i], inv))));
      packed |= (uint32_t)(uint8_t)(int8_t)c << (8 * i);
    }
  }
  int8_t* dst = (is_k ? k8 : q8) + off;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint32_t*>(dst) = packed;
  } else {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
  }
  if (lane == 0) *scale = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
}

}  // namespace

cudaError_t launch_quant_qk(const uint16_t* q, const uint16_t* k, int8_t* q8, int8_t* k8, float* sq, float* sk,
                            int H, int S, int d, int stride, cudaStream_t stream) {
  const long long warps = 2LL * H * stride;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  if (d == 64)
    quant_rows_kernel<64><<<grid, 256, 0, stream>>>(q, k, q8, k8, sq, sk, H, S, stride);
  else
    quant_rows_kernel<128><<<grid, 256, 0, stream>>>(q, k, q8, k8, sq, sk, H, S, stride);
  return cudaGetLastError();
}

}  // namespace h3
