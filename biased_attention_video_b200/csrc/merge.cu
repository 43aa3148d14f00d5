// Merge of normalised partition results ("Flash Partitions for H3 native
// temporal alignment", section 4 "Why log-sum-exp is necessary"): partition i
// has output O_i (already divided by its own normaliser), natural-log
// normaliser L_i and multiplier w_i (log w_i given; -inf for w_i = 0);
//     adjusted_L_i = L_i + log w_i,  L = logsumexp_i adjusted_L_i,
//     O = sum_i exp(adjusted_L_i - L) O_i.
// A row whose adjusted normalisers are all -inf gets O = 0 and L = -inf.
//
// HBM-bound: specialised on the number of partitions; each thread merges 16
// bytes of one row (all its loads issued first) and writes them back.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace h3 {
namespace {

// NP partitions; each thread merges 8 consecutive elements (16 bytes) of one
// row, D / 8 threads per row, all its loads issued before the arithmetic.
template <int D, int NP>
__global__ void __launch_bounds__(256) merge_kernel(MergeParts parts, long long rows, uint16_t* __restrict__ o,
                                                    float* __restrict__ lse) {
  constexpr int kThreadsPerRow = D / 8;
  constexpr int kRowsPerBlock = 256 / kThreadsPerRow;
  const long long row = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kThreadsPerRow;
  const int sub = threadIdx.x % kThreadsPerRow;
  if (row >= rows) return;
  uint4 v[NP];
  float adj[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    v[i] = __ldg(reinterpret_cast<const uint4*>(parts.o[i] + row * D) + sub);
    adj[i] = __ldg(parts.lse[i] + row) + parts.log_w[i];
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < NP; ++i) m = fmaxf(m, adj[i]);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float L = -INFINITY;
  if (m > -INFINITY) {
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < NP; ++i) s += expf(adj[i] - m);
    L = m + logf(s);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float w = expf(adj[i] - L);
      const uint32_t words[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        acc[2 * h] = fmaf(w, __uint_as_float(words[h] << 16), acc[2 * h]);
        acc[2 * h + 1] = fmaf(w, __uint_as_float(words[h] & 0xFFFF0000u), acc[2 * h + 1]);
      }
    }
  }
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
    out[h] = *reinterpret_cast<uint32_t*>(&b);
  }
  reinterpret_cast<uint4*>(o + row * D)[sub] = make_uint4(out[0], out[1], out[2], out[3]);
  if (lse != nullptr && sub == 0) lse[row] = L;
}

template <int D>
cudaError_t launch_merge_d(const MergeParts& parts, long long rows, uint16_t* o, float* lse, cudaStream_t stream) {
  constexpr int kRowsPerBlock = 256 / (D / 8);
  const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  switch (parts.n) {
    case 1: merge_kernel<D, 1><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 2: merge_kernel<D, 2><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 3: merge_kernel<D, 3><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 4: merge_kernel<D, 4><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 5: merge_kernel<D, 5><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 6: merge_kernel<D, 6><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    case 7: merge_kernel<D, 7><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
    default: merge_kernel<D, kMaxMergeParts><<<grid, 256, 0, stream>>>(parts, rows, o, lse); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeParts& parts, long long rows, int d, uint16_t* o, float* lse,
                         cudaStream_t stream) {
  if (rows <= 0 || parts.n < 1 || parts.n > kMaxMergeParts) return rows <= 0 ? cudaSuccess : cudaErrorInvalidValue;
  return d == 64 ? launch_merge_d<64>(parts, rows, o, lse, stream) : launch_merge_d<128>(parts, rows, o, lse, stream);
}

}  // namespace h3
