// Pooled tail term ("H3 SLA Attention", inputs table, tail_correction): the
// video key blocks that top-k left out of a query block's list enter its
// softmax through one pooled term instead of being dropped, scored from the
// pooled centroids routing already computed.  Per video query block i:
//     Lt_i = log sum_{j dropped} n_j exp(s_ij),   s_ij = Qp_i . Kp_j / sqrt(d)
//     Ot_i = sum_{j dropped} n_j exp(s_ij - Lt_i) Vp_j
// (n_j valid rows of block j, Vp_j its mean V row; no temporal penalty, as
// routing sees none), then every row of block i merges (Ot_i, Lt_i) with its
// exact routed result as one more partition of weight 1.
//
// Four kernels:
//  1. pool_vt_kernel: mean V row of every video block, written transposed in
//     bf16 (vpt[h][c][j]) as the GEMM's K-major B operand.
//  2. tail_weights_kernel: one warp per (head, query block): from the fp32
//     pooled scores routing left in the workspace and the routed list, the
//     weights W_ij = n_j exp(s_ij - M_i) of the dropped blocks (0 for routed
//     ones) in bf16, and the row's log mass Lt_i = M_i + log sum_j W_ij.
//  3. tail_gemm_kernel: Ot = diag(1 / sum_j W_ij) W Vp on the tensor cores
//     (tcgen05, M = 128 query blocks, N = d, K = key blocks in chunks of 64).
//  4. tail_merge_kernel: per row of a video query block, logsumexp merge of
//     (O, LSE) with (Ot_i, Lt_i), in place.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_value(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// ------------------------------------------------------------------ 1. pooled V
// One warp per (head, video block j < ldk): lanes own 8 columns of a row, the
// warp's rows are summed in fp32, the mean goes to vpt[h][c][j]; j >= n_video
// is zero padding.
template <int D>
__global__ void __launch_bounds__(256) pool_vt_kernel(const uint16_t* __restrict__ v, uint16_t* __restrict__ vpt,
                                                      int H, int S, int first_block, int n_video, int ldk) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  const long long warp_id = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (warp_id >= (long long)H * ldk) return;
  const int h = (int)(warp_id / ldk), j = (int)(warp_id % ldk);
  const int chunk = lane % kLanesPerRow, rsub = lane / kLanesPerRow;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int nrows = 0;
  if (j < n_video) {
    const int row0 = (first_block + j) * kBlock;
    nrows = min(kBlock, S - row0);
    const uint4* src = reinterpret_cast<const uint4*>(v + ((size_t)h * S + row0) * D) + chunk;
    for (int r = rsub; r < nrows; r += kRowsPerPass) {
      const uint4 x = __ldg(src + (size_t)r * kLanesPerRow);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __uint_as_float(w[q] << 16);
        acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int o = kLanesPerRow; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], o);
  if (rsub == 0) {
    const float inv = nrows > 0 ? 1.0f / (float)nrows : 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) vpt[((size_t)h * D + chunk * 8 + e) * ldk + j] = bf16_bits(acc[e] * inv);
  }
}

// ------------------------------------------------------------------ 2. weights
// One warp per (head, video query block i); a per-warp bitmap of the routed
// blocks in shared memory ((n_video + 31) / 32 words).
__global__ void __launch_bounds__(256) tail_weights_kernel(const float* __restrict__ scores, int ldc,
                                                           const int32_t* __restrict__ sel, int k, int H, int S,
                                                           int first_block, int n_video, float scale,
                                                           uint16_t* __restrict__ w, int ldk,
                                                           float* __restrict__ lt, float* __restrict__ inv_sum) {
  extern __shared__ uint32_t tw_bits[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= (long long)H * n_video) return;  // warp-uniform
  const int words = (n_video + 31) >> 5;
  uint32_t* kept = tw_bits + (size_t)warp * words;
  for (int i = lane; i < words; i += 32) kept[i] = 0u;
  __syncwarp();
  const int32_t* lst = sel + (size_t)row * k;
  for (int t = lane; t < k; t += 32) {
    const int j = lst[t] - first_block;
    if (j >= 0 && j < n_video) atomicOr(kept + (j >> 5), 1u << (j & 31));
  }
  __syncwarp();
  const float* srow = scores + (size_t)row * ldc;
  const int last_rows = S - (first_block + n_video - 1) * kBlock;  // valid rows of the last block
  const float log_full = __logf((float)kBlock), log_last = __logf((float)last_rows);
  auto logit = [&](int j) -> float {  // s_ij + log n_j of a dropped block, -inf for a routed one
    if ((kept[j >> 5] >> (j & 31)) & 1u) return -INFINITY;
    return fmaf(srow[j], scale, j == n_video - 1 ? log_last : log_full);
  };
  // unrolled so that several score loads are in flight per lane
  float m = -INFINITY;
#pragma unroll 8
  for (int j = lane; j < n_video; j += 32) m = fmaxf(m, logit(j));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  uint16_t* wrow = w + (size_t)row * ldk;
  float sum = 0.0f;
#pragma unroll 8
  for (int j = lane; j < ldk; j += 32) {
    uint16_t b = 0;
    if (j < n_video && m > -INFINITY) {
      const float x = logit(j);
      if (x > -INFINITY) b = bf16_bits(__expf(x - m));
    }
    wrow[j] = b;
    sum += bf16_value(b);  // the GEMM sees the rounded weights
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane == 0) {
    lt[row] = sum > 0.0f ? m + __logf(sum) : -INFINITY;
    inv_sum[row] = sum > 0.0f ? 1.0f / sum : 0.0f;
  }
}

// ------------------------------------------------------------------ 3. GEMM
constexpr int kTM = 128;  // query blocks per tile
constexpr int kTStages = 2;

__device__ __forceinline__ bool tail_wait(uint64_t* bar, uint32_t parity, int* status) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      if (now - t0 > 2000000000ull) {
        if (status != nullptr) atomicCAS(status, 0, kStatusTimeout);
        return false;
      }
    }
  }
}

template <int D>
struct TailGemmLayout {
  static constexpr int kStageA = kTM * 128;  // one 64-element (128-byte) K chunk of W
  static constexpr int kStageB = D * 128;    // the same K chunk of Vp^T
  static constexpr int kStageBytes = kStageA + kStageB;
  static constexpr int kBars = kTStages * kStageBytes;
  static constexpr int kSmem = 1024 + kBars + 64;
};

// ot[h][i][:] = bf16(inv_sum[h][i] * sum_j w[h][i][j] vpt[h][:][j]) for query
// blocks i in [m0, m0 + 128) of head h.
template <int D>
__global__ void __launch_bounds__(128) tail_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                        const __grid_constant__ CUtensorMap tm_v,
                                                        uint16_t* __restrict__ ot, const float* __restrict__ inv_sum,
                                                        int n_video, int n_chunks, int* status) {
  using L = TailGemmLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + kTStages;
  uint64_t* done = empty + kTStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kTM, h = blockIdx.y;
  if (tid == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, D);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    uint32_t issued[kTStages] = {0, 0};
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c % kTStages;
      const uint32_t ph = (uint32_t)(c / kTStages) & 1u;
      if (!tail_wait(empty + s, ph ^ 1u, status)) break;
      uint8_t* st = smem + s * L::kStageBytes;
      mbar_arrive_expect_tx(full + s, L::kStageBytes);
      tma_load_3d(st, &tm_w, full + s, c * 64, m0, h);
      tma_load_3d(st + L::kStageA, &tm_v, full + s, c * 64, 0, h);
      ++issued[s];
    }
    for (int s = 0; s < kTStages; ++s)
      if (issued[s]) tail_wait(full + s, (issued[s] - 1) & 1u, status);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTM, D, 0, 0);
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c % kTStages;
      const uint32_t ph = (uint32_t)(c / kTStages) & 1u;
      if (!tail_wait(full + s, ph, status)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * L::kStageBytes), b = a + L::kStageA;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_ss(tmem, sw128_desc(a + kk * 32, 16, 1024), sw128_desc(b + kk * 32, 16, 1024), kIdesc,
                (c > 0 || kk > 0) ? 1u : 0u);
      umma_commit(empty + s);
    }
    umma_commit(done);
  }
  // epilogue: thread = query block; TMEM row -> scaled bf16 row of ot
  const bool got = tail_wait(done, 0, status);
  if (__all_sync(0xFFFFFFFFu, got)) {
    tc_fence_after();
    const int i = m0 + warp * 32 + lane;
    const float sc = i < n_video ? __ldg(inv_sum + (size_t)h * n_video + i) : 0.0f;
    uint16_t* row = ot + ((size_t)h * n_video + (i < n_video ? i : 0)) * D;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t v[32];
      __syncwarp();
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + cc * 32, v);
      tmem_wait_ld();
      if (i < n_video) {
        uint32_t packed[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[2 * t]) * sc, __uint_as_float(v[2 * t + 1]) * sc);
          packed[t] = *reinterpret_cast<uint32_t*>(&b);
        }
        uint4* dst = reinterpret_cast<uint4*>(row + cc * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t) dst[t] = make_uint4(packed[4 * t], packed[4 * t + 1], packed[4 * t + 2], packed[4 * t + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, D);
  }
}

// ------------------------------------------------------------------ 4. merge
// D / 8 threads per row of a video query block, 16 bytes each: O and LSE of
// the row merged in place with the block's tail partition.  Each thread takes
// kMergeRows rows (a block's passes kRowsPerPass rows apart), loading all of
// them before merging any, so that several 16-byte loads are in flight.
constexpr int kMergeRows = 4;

template <int D>
__global__ void __launch_bounds__(256) tail_merge_kernel(uint16_t* __restrict__ o, float* __restrict__ lse,
                                                         const uint16_t* __restrict__ ot,
                                                         const float* __restrict__ lt, int H, int S,
                                                         int first_block, int n_video) {
  constexpr int kThreadsPerRow = D / 8;
  constexpr int kRowsPerPass = 256 / kThreadsPerRow;
  const long long video_rows = (long long)S - (long long)first_block * kBlock;
  const long long total = (long long)H * video_rows;
  const long long t0 = (long long)blockIdx.x * kRowsPerPass * kMergeRows + threadIdx.x / kThreadsPerRow;
  const int sub = threadIdx.x % kThreadsPerRow;
  uint4 a[kMergeRows], b[kMergeRows];
  float la[kMergeRows], lb[kMergeRows];
  long long orow[kMergeRows];
#pragma unroll
  for (int k = 0; k < kMergeRows; ++k) {
    const long long t = t0 + (long long)k * kRowsPerPass;
    orow[k] = -1;
    if (t < total) {
      const int h = (int)(t / video_rows);
      const long long r = (long long)first_block * kBlock + t % video_rows;  // sequence row
      const int i = (int)(r / kBlock) - first_block;                         // its video query block
      orow[k] = (long long)h * S + r;
      a[k] = *(reinterpret_cast<const uint4*>(o + orow[k] * D) + sub);
      b[k] = __ldg(reinterpret_cast<const uint4*>(ot + ((size_t)h * n_video + i) * D) + sub);
      la[k] = lse[orow[k]];
      lb[k] = __ldg(lt + (size_t)h * n_video + i);
    }
  }
#pragma unroll
  for (int k = 0; k < kMergeRows; ++k) {
    if (orow[k] < 0) continue;
    const float m = fmaxf(la[k], lb[k]);
    if (m == -INFINITY) continue;  // nothing on either side: leave the row as it is
    const float L = m + __logf(__expf(la[k] - m) + __expf(lb[k] - m));
    const float wa = __expf(la[k] - L), wb = __expf(lb[k] - L);
    const uint32_t aw[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, bw[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = fmaf(wa, __uint_as_float(aw[q] << 16), wb * __uint_as_float(bw[q] << 16));
      const float hi = fmaf(wa, __uint_as_float(aw[q] & 0xFFFF0000u), wb * __uint_as_float(bw[q] & 0xFFFF0000u));
      __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
      out[q] = *reinterpret_cast<uint32_t*>(&v);
    }
    *(reinterpret_cast<uint4*>(o + orow[k] * D) + sub) = make_uint4(out[0], out[1], out[2], out[3]);
    if (sub == 0) lse[orow[k]] = L;
  }
}

}  // namespace

TailScratch tail_scratch_layout(int H, int d, int n_video) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  TailScratch t;
  t.ldk = (n_video + 63) / 64 * 64;
  t.w = 0;
  t.vpt = up((size_t)H * n_video * t.ldk * 2);
  t.ot = t.vpt + up((size_t)H * d * t.ldk * 2);
  t.lt = t.ot + up((size_t)H * n_video * d * 2);
  t.inv_sum = t.lt + up((size_t)H * n_video * 4);
  t.total = t.inv_sum + up((size_t)H * n_video * 4);
  return t;
}

cudaError_t launch_tail(const uint16_t* v, const float* scores, size_t ldc, const int32_t* kv_sel, int kk, int H,
                        int S, int d, int first_block, int n_video, uint16_t* o, float* lse, void* scratch,
                        int* status, cudaStream_t stream) {
  const TailScratch t = tail_scratch_layout(H, d, n_video);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint16_t* w = reinterpret_cast<uint16_t*>(base + t.w);
  uint16_t* vpt = reinterpret_cast<uint16_t*>(base + t.vpt);
  uint16_t* ot = reinterpret_cast<uint16_t*>(base + t.ot);
  float* lt = reinterpret_cast<float*>(base + t.lt);
  float* inv_sum = reinterpret_cast<float*>(base + t.inv_sum);
  const int ldk = (int)t.ldk;
  // 1. pooled V
  const long long pwarps = (long long)H * ldk;
  if (d == 64)
    pool_vt_kernel<64><<<(unsigned)((pwarps + 7) / 8), 256, 0, stream>>>(v, vpt, H, S, first_block, n_video, ldk);
  else
    pool_vt_kernel<128><<<(unsigned)((pwarps + 7) / 8), 256, 0, stream>>>(v, vpt, H, S, first_block, n_video, ldk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. weights (8 warps per block, a bitmap per warp)
  const int words = (n_video + 31) / 32;
  const size_t wsmem = (size_t)8 * words * 4;
  e = cudaFuncSetAttribute(tail_weights_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsmem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)H * n_video;
  tail_weights_kernel<<<(unsigned)((rows + 7) / 8), 256, wsmem, stream>>>(
      scores, (int)ldc, kv_sel, kk, H, S, first_block, n_video, 1.0f / sqrtf((float)d), w, ldk, lt, inv_sum);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. GEMM on the tensor cores
  CUtensorMap tw, tv;
  if (!encode_bf16_3d(&tw, w, ldk, n_video, H, 64, kTM) || !encode_bf16_3d(&tv, vpt, ldk, d, H, 64, d))
    return cudaErrorInvalidValue;
  const dim3 grid((n_video + kTM - 1) / kTM, H);
  if (d == 64) {
    e = cudaFuncSetAttribute(tail_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TailGemmLayout<64>::kSmem);
    if (e == cudaSuccess)
      tail_gemm_kernel<64><<<grid, 128, TailGemmLayout<64>::kSmem, stream>>>(tw, tv, ot, inv_sum, n_video,
                                                                             ldk / 64, status);
  } else {
    e = cudaFuncSetAttribute(tail_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TailGemmLayout<128>::kSmem);
    if (e == cudaSuccess)
      tail_gemm_kernel<128><<<grid, 128, TailGemmLayout<128>::kSmem, stream>>>(tw, tv, ot, inv_sum, n_video,
                                                                               ldk / 64, status);
  }
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 4. merge into O / LSE
  const long long mrows = (long long)H * ((long long)S - (long long)first_block * kBlock);
  const int rows_per_block = 256 / (d / 8) * kMergeRows;
  const unsigned mgrid = (unsigned)((mrows + rows_per_block - 1) / rows_per_block);
  if (mgrid > 0) {
    if (d == 64)
      tail_merge_kernel<64><<<mgrid, 256, 0, stream>>>(o, lse, ot, lt, H, S, first_block, n_video);
    else
      tail_merge_kernel<128><<<mgrid, 256, 0, stream>>>(o, lse, ot, lt, H, S, first_block, n_video);
  }
  return cudaGetLastError();
}

}  // namespace h3
