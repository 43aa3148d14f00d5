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
// HBM-bound: d / 8 lanes per row with one 16-byte load each, eight rows per
// warp with all loads issued before the arithmetic, one 64-row block per CTA.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace h3 {
namespace {

constexpr int kRowsPerWarp = 8;  // rows per warp, all loads issued first (8 warps: one 64-row block)

// grid (n_blocks, 2 H): CTA (b, t H + h) quantises rows [64 b, 64 b + 64) of
// head h of Q (t = 0) or K (t = 1).  D / 8 lanes per row (16 bytes each):
// 32 / (D / 8) rows per pass.
template <int D>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                         int8_t* __restrict__ q8, int8_t* __restrict__ k8,
                                                         float* __restrict__ sq, float* __restrict__ sk, int H, int S,
                                                         int stride) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  constexpr int kPasses = kRowsPerWarp / kRowsPerPass;
  const int lane = threadIdx.x & 31;
  const int sub = lane % kLanesPerRow;  // 16-byte chunk of the row
  const bool is_k = (int)blockIdx.y >= H;
  const int h = is_k ? (int)blockIdx.y - H : (int)blockIdx.y;
  const int r0 = (int)blockIdx.x * 64 + (threadIdx.x >> 5) * kRowsPerWarp + lane / kLanesPerRow;
  const uint16_t* src = (is_k ? k : q) + (size_t)h * S * D;
  int8_t* dst = (is_k ? k8 : q8) + (size_t)h * S * D;
  float* scale = (is_k ? sk : sq) + (size_t)h * stride;
  uint4 w[kPasses];
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int r = r0 + i * kRowsPerPass;
    w[i] = r < S ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * D) + sub) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int r = r0 + i * kRowsPerPass;
    const uint32_t x[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
    float v[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(x[e] << 16);
      v[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
    }
    // |x| of finite floats orders like its bit pattern; max over the row's lanes
    uint32_t amax = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = max(amax, __float_as_uint(v[e]) & 0x7FFFFFFFu);
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float a = __uint_as_float(amax);
    uint2 packed = make_uint2(0u, 0u);
    if (a > 0.0f) {
      const float inv = __fdiv_rn(127.0f, a);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        // rint by the exponent trick: for |t| < 2^22, t + (2^23 + 2^22) rounds
        // t to the nearest integer, ties to even, and that integer sits in
        // the low mantissa bits (t = 0 * inf = NaN, from a subnormal a, is
        // taken as 0)
        const float t = __fmul_rn(v[e], inv);
        const float tc = t != t ? 0.0f : fminf(fmaxf(t, -127.0f), 127.0f);
        const int c = __float_as_int(__fadd_rn(tc, 12582912.0f)) - 0x4B400000;
        const uint32_t b = (uint32_t)(uint8_t)(int8_t)c << (8 * (e & 3));
        if (e < 4) packed.x |= b;
        else packed.y |= b;
      }
    }
    if (r < S) reinterpret_cast<uint2*>(dst + (size_t)r * D)[sub] = packed;
    if (sub == 0) scale[r] = r < S && a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
  }
}

}  // namespace

cudaError_t launch_quant_qk(const uint16_t* q, const uint16_t* k, int8_t* q8, int8_t* k8, float* sq, float* sk,
                            int H, int S, int d, int stride, cudaStream_t stream) {
  if (stride % 64 != 0 || 2LL * H > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)(stride / 64), (unsigned)(2 * H));
  if (d == 64)
    quant_rows_kernel<64><<<grid, 256, 0, stream>>>(q, k, q8, k8, sq, sk, H, S, stride);
  else
    quant_rows_kernel<128><<<grid, 256, 0, stream>>>(q, k, q8, k8, sq, sk, H, S, stride);
  return cudaGetLastError();
}

}  // namespace h3
