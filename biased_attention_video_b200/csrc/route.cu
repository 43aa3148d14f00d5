// Pooled-score routing ("H3 SLA Attention", "How it works": every query block
// is scored against every key block with one small pooled matmul and only the
// top 1 - sparsity_ratio fraction is kept).
//
// Three kernels:
//  1. pool_split_kernel: mean of every video block of Q and K (fp32 sums of the
//     bf16 rows), written as three bf16 parts x = h + m + l (h = bf16(x),
//     m = bf16(x - h), l = bf16(x - h - m): together the 24 significant bits of
//     the fp32 mean), rows [h | h | m | h | m | l] for Q and [h | m | h | l | m | h]
//     for K.
//  2. score_gemm_kernel: per head, scores = Qs . Ks^T over the concatenated
//     6d-long rows, i.e. Qh.Kh + Qh.Km + Qm.Kh + Qh.Kl + Qm.Km + Ql.Kh -- every
//     product of the pooled centroids' parts down to relative order 2^-16 (the
//     dropped ones are below 2^-24), each exact in fp32, accumulated in fp32 on
//     the tensor cores (tcgen05.mma kind::f16, fp32 accumulation in TMEM).
//  3. topk_kernel: one warp per (head, query block): the k best key blocks,
//     ties to the lower block, listed in ascending order.
// The 1/sqrt(d) logit scale is a positive constant and does not change the
// order, so it is not applied.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

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

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One warp per (tensor, head, video block).  Output row layout (kSplitParts d
// bf16): Q: [h | h | m | h | m | l], K: [h | m | h | l | m | h], so that the row
// dot product of the two concatenations is Qh.Kh + Qh.Km + Qm.Kh + Qh.Kl +
// Qm.Km + Ql.Kh.
template <int D>
__global__ void __launch_bounds__(256) pool_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                         uint16_t* __restrict__ qs, uint16_t* __restrict__ ks, int H,
                                                         int S, int first_block, int n_video) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  constexpr int kPasses = kBlock / kRowsPerPass;
  const long long warp_id = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long per_tensor = (long long)H * n_video;
  if (warp_id >= 2 * per_tensor) return;
  const int t = (int)(warp_id / per_tensor);
  const long long rem = warp_id % per_tensor;
  const int h = (int)(rem / n_video);
  const int vb = (int)(rem % n_video);
  const int row0 = (first_block + vb) * kBlock;
  const int nrows = min(kBlock, S - row0);
  const int chunk = lane % kLanesPerRow;
  const int rsub = lane / kLanesPerRow;
  const uint16_t* x = t == 0 ? q : k;
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)h * S + row0) * D) + chunk;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (nrows == kBlock) {
    constexpr int kBatch = 8;
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
    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // the differences are exact in fp32: each part takes the next 8 significant bits
      const float a = acc[2 * i] * inv, b = acc[2 * i + 1] * inv;
      const float ah = __bfloat162float(__float2bfloat16_rn(a)), bh = __bfloat162float(__float2bfloat16_rn(b));
      const float am = __bfloat162float(__float2bfloat16_rn(a - ah));
      const float bm = __bfloat162float(__float2bfloat16_rn(b - bh));
      hw[i] = bf16x2_bits(ah, bh);
      mw[i] = bf16x2_bits(am, bm);
      lw[i] = bf16x2_bits((a - ah) - am, (b - bh) - bm);
    }
    const uint4 hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    const uint4 mv = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    const uint4 lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    uint16_t* dst_row = (t == 0 ? qs : ks) + ((size_t)h * n_video + vb) * (kSplitParts * D) + chunk * 8;
    const uint4 q_parts[kSplitParts] = {hv, hv, mv, hv, mv, lv};
    const uint4 k_parts[kSplitParts] = {hv, mv, hv, lv, mv, hv};
#pragma unroll
    for (int part = 0; part < kSplitParts; ++part)
      *reinterpret_cast<uint4*>(dst_row + part * D) = t == 0 ? q_parts[part] : k_parts[part];
  }
}


// ----------------------------------------------------------- score GEMM
// Persistent: one CTA per SM walks the 128 x 256 output tiles (head, query
// blocks, key blocks) in steps of the grid size.  Warp 0 loads 64-element K
// chunks of A and B through a three-stage TMA ring, warp 1 issues the MMAs into
// one of two TMEM accumulators (2 x 256 columns), and warps 2..5 write the
// other accumulator's scores out, so the epilogue of tile i overlaps the MMAs
// of tile i + 1.  Each epilogue warp stages 32 rows x 32 scores in shared
// memory (128-byte swizzle, two buffers) and stores them with one TMA tile
// store, which also drops the rows and columns past the video blocks.  The
// scores' HBM writes bound it (4 B per score).
constexpr int kGemmThreads = 192;
constexpr int kGM = 128;                    // query blocks per tile (UMMA M)
constexpr int kGN = 256;                    // key blocks per tile (UMMA N)
constexpr int kGStages = 3;
constexpr int kGStageA = kGM * 128;         // one 64-element (128-byte) K chunk of A
constexpr int kGStageB = kGN * 128;
constexpr int kGStageBytes = kGStageA + kGStageB;
constexpr int kGEpi = kGStages * kGStageBytes;  // epilogue staging: 4 warps x 2 x 4 KB
constexpr int kGEpiBytes = 4 * 2 * 4096;
constexpr int kGBars = kGEpi + kGEpiBytes;
constexpr int kGNumBars = 2 * kGStages + 5;  // full, empty, acc_full[2], acc_empty[2], drain
constexpr int kGSmem = 1024 + kGBars + kGNumBars * 8 + 16;
constexpr uint32_t kGTmemCols = 2 * kGN;

// Bounded wait with CTA-wide abort (on give-up: abort flag and status word).
__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      if (now - t0 > 2000000000ull) {
        *abort = 1;
        if (status != nullptr) atomicCAS(status, 0, kStatusTimeout);
        return false;
      }
    }
  }
}

// Bounded wait for in-flight async work before exit (ignores the abort flag).
__device__ __forceinline__ void gemm_drain(uint64_t* bar, uint32_t parity, int* status) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      if (now - t0 > 2000000000ull) {
        if (status != nullptr) atomicCAS(status, 0, kStatusTimeout);
        return;
      }
    }
  }
}

// scores[h][i][j] for every video query block i and video key block j of
// every head, written through tm_c (fp32 [H][n_video] rows of pitch ldc, TMA
// store map).  Tile t covers head t / (n_tm n_tn), query blocks
// [128 ((t / n_tn) % n_tm), +128) and key blocks [256 (t % n_tn), +256); rows
// past n_video read as zero (TMA fill) and are not stored.
__global__ void __launch_bounds__(kGemmThreads, 1)
    score_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_c, int n_video, int n_chunks, int n_tm, int n_tn,
                      int n_tiles, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGBars);
  uint64_t* empty = full + kGStages;
  uint64_t* acc_full = empty + kGStages;  // [2]: accumulator b holds a finished tile
  uint64_t* acc_empty = acc_full + 2;     // [2]: the epilogue has read accumulator b
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int per_head = n_tm * n_tn;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t issued[kGStages] = {};
      uint32_t q = 0;  // K chunks issued so far, over all tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int h = t / per_head, m0 = ((t / n_tn) % n_tm) * kGM, n0 = (t % n_tn) * kGN;
        for (int c = 0; c < n_chunks; ++c, ++q) {
          const int s = (int)(q % kGStages);
          const uint32_t ph = (q / kGStages) & 1u;
          if (!gemm_wait(empty + s, ph ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kGStageBytes;
          mbar_arrive_expect_tx(full + s, kGStageBytes);
          tma_load_3d(st, &tm_a, full + s, c * 64, m0, h);
          tma_load_3d(st + kGStageA, &tm_b, full + s, c * 64, n0, h);
          ++issued[s];
        }
      }
      // every issued load lands before the CTA may exit
      for (int s = 0; s < kGStages; ++s)
        if (issued[s]) gemm_drain(full + s, (issued[s] - 1) & 1u, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16_f32(kGM, kGN, 0, 0);
      uint32_t q = 0;
      bool ok = true;
      int i = 0;  // tiles of this CTA so far
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
        const int b = i & 1;
        // accumulator b is free once the epilogue has read its previous tile
        if (!gemm_wait(acc_empty + b, ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kGN);
        for (int c = 0; c < n_chunks; ++c, ++q) {
          const int s = (int)(q % kGStages);
          const uint32_t ph = (q / kGStages) & 1u;
          if (!gemm_wait(full + s, ph, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * kGStageBytes), bb = a + kGStageA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(d_tmem, sw128_desc(a + kk * 32, 16, 1024), sw128_desc(bb + kk * 32, 16, 1024), kIdesc,
                    (c > 0 || kk > 0) ? 1u : 0u);
          umma_commit(empty + s);
        }
        if (ok) umma_commit(acc_full + b);
      }
      // every issued MMA completes before TMEM is released
      umma_commit(drain);
      gemm_drain(drain, 0, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = query block row (TMEM lane); warp w reads lanes 32 (w % 4)..
    // and writes each 32 x 32 block of scores through shared memory: row r at
    // byte 128 r, its 16-byte chunk c at chunk c ^ (r & 7) (the 128-byte
    // swizzle of the store's tensor map; conflict-free for the warp)
    const int quarter = warp & 3;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    uint8_t* stage = smem + kGEpi + (warp - 2) * 2 * 4096;
    uint32_t n_st = 0;  // 32 x 32 blocks staged by this warp
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      if (!__all_sync(0xFFFFFFFFu, gemm_wait(acc_full + b, (uint32_t)(i >> 1) & 1u, abort_flag, status))) break;
      tc_fence_after();
      const int h = t / per_head, m0 = ((t / n_tn) % n_tm) * kGM, n0 = (t % n_tn) * kGN;
      const int row0 = m0 + quarter * 32;
#pragma unroll 1
      for (int cc = 0; cc < kGN / 32; ++cc) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_addr + (uint32_t)(b * kGN + cc * 32), v);
        tmem_wait_ld();
        const int j0 = n0 + cc * 32;
        if (row0 >= n_video || j0 >= n_video) continue;  // warp-uniform: nothing of the block is stored
        uint8_t* buf = stage + (n_st & 1u) * 4096;
        // the store that read this buffer two blocks ago is done with it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        uint8_t* my_row = buf + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(my_row + ((c ^ (lane & 7)) << 4)) =
              make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the bulk store
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_c, buf, j0, row0, h);
          bulk_commit();
        }
        ++n_st;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + b);
    }
    // every store has written global memory before the CTA exits
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGTmemCols);
  }
}


// ----------------------------------------------------------------- top-k
// Per-warp shared memory (32-bit words): the row's scores (ldc), a 256-bin
// histogram, candidate indices (16-bit) and a bitmap of chosen candidates.
__host__ __device__ __forceinline__ int topk_warp_words(int n_video, int ldc) {
  return (ldc + 256 + (n_video + 1) / 2 + (n_video + 31) / 32 + 3) & ~3;
}

// One warp per (head, video query block).  Selection: the row is binned
// linearly between its minimum and maximum (a monotone map, equal scores share
// a bin); the bin holding the k-th best score is found from the top of a
// 256-bin histogram; every score in a higher bin is taken, and the candidates
// in that bin are ranked exactly by (score descending, block ascending).
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel,
                                                   int rows, int n_video, int ldc, int k, int first_video_block) {
  extern __shared__ float4 tk_smem4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;  // warp-uniform
  const int words = topk_warp_words(n_video, ldc);
  uint32_t* base = reinterpret_cast<uint32_t*>(tk_smem4) + (size_t)warp * words;
  float* s = reinterpret_cast<float*>(base);
  uint32_t* hist = base + ldc;
  uint16_t* cand = reinterpret_cast<uint16_t*>(hist + 256);
  uint32_t* chosen = hist + 256 + (n_video + 1) / 2;
  const unsigned full = 0xFFFFFFFFu;
  const uint32_t lt_mask = (1u << lane) - 1u;

  const float* src = scores + (size_t)row * ldc;
  for (int j = lane * 4; j < n_video; j += 128) {
    const float4 v = *reinterpret_cast<const float4*>(src + j);
    *reinterpret_cast<float4*>(s + j) = v;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0u;
  for (int w = lane; w < (n_video + 31) / 32; w += 32) chosen[w] = 0u;
  __syncwarp();
  float lo = INFINITY, hi = -INFINITY;
  for (int j = lane; j < n_video; j += 32) {
    lo = fminf(lo, s[j]);
    hi = fmaxf(hi, s[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(full, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(full, hi, o));
  }
  const float bscale = hi > lo ? 256.0f / (hi - lo) : 0.0f;
  auto bin_of = [&](float x) -> int { return min(255, (int)((x - lo) * bscale)); };
  for (int j = lane; j < n_video; j += 32) atomicAdd(hist + bin_of(s[j]), 1u);
  __syncwarp();
  // bin T holding the k-th best: lane l owns bins 255-8l .. 248-8l (descending)
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    c[e] = hist[255 - 8 * lane - e];
    sum += c[e];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(full, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - sum;
  const bool here = excl < (uint32_t)k && (uint32_t)k <= incl;
  const int src_lane = __ffs(__ballot_sync(full, here)) - 1;
  int tbin = 0;
  uint32_t greater = 0;
  if (here) {
    uint32_t cum = excl;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (cum + c[e] >= (uint32_t)k) {
        tbin = 255 - 8 * lane - e;
        greater = cum;
        break;
      }
      cum += c[e];
    }
  }
  tbin = __shfl_sync(full, tbin, src_lane);
  greater = __shfl_sync(full, greater, src_lane);
  const int need = k - (int)greater;
  // candidates (scores in bin tbin), gathered in ascending block order
  int n_cand = 0;
  for (int jb = 0; jb < n_video; jb += 32) {
    const int j = jb + lane;
    const bool is_c = j < n_video && bin_of(s[j]) == tbin;
    const uint32_t m = __ballot_sync(full, is_c);
    if (is_c) cand[n_cand + __popc(m & lt_mask)] = (uint16_t)j;
    n_cand += __popc(m);
  }
  __syncwarp();
  // exact rank among candidates: (score descending, block ascending)
  for (int e = lane; e < n_cand; e += 32) {
    const int je = cand[e];
    const float ve = s[je];
    int rank = 0;
    for (int f = 0; f < n_cand; ++f) {
      const int jf = cand[f];
      const float vf = s[jf];
      rank += (vf > ve || (vf == ve && jf < je)) ? 1 : 0;
    }
    if (rank < need) atomicOr(chosen + (je >> 5), 1u << (je & 31));
  }
  __syncwarp();
  int32_t* dst = sel + (size_t)row * k;
  int pos = 0;
  for (int jb = 0; jb < n_video; jb += 32) {
    const int j = jb + lane;
    bool take = false;
    if (j < n_video) {
      const int b = bin_of(s[j]);
      take = b > tbin || (b == tbin && ((chosen[j >> 5] >> (j & 31)) & 1u));
    }
    const uint32_t m = __ballot_sync(full, take);
    const int slot = pos + __popc(m & lt_mask);
    if (take && slot < k) dst[slot] = first_video_block + j;
    pos += __popc(m);
  }
}

// Register-resident top-k for rows of at most 32 NPL scores (one warp per
// (head, video query block)); the same selection as topk_kernel: the k
// highest scores, ties to the lower block, listed in ascending block order.
// Lane l holds the scores j = l + 32 i (i < NPL) as order-preserving integer
// keys (-0 folded into +0 first, so equal floats give equal keys; padding
// past n_video gets key 0, below every real key).  The candidates are always
// a contiguous key range [alo, ahi]: each level bins that range into 256
// bins of 2^shift keys, takes every key above the bin that holds the next
// needed key, and narrows the range to that bin.  shift drops by 8 per
// level, so after at most four levels the range is one key and its keys go
// by ascending block; shared memory holds only the warp's histogram.
template <int NPL>
__global__ void __launch_bounds__(256, 2) topk_reg_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel,
                                                          int rows, int n_video, int ldc, int k, int first_video_block) {
  __shared__ uint32_t hist_all[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;  // warp-uniform
  uint32_t* hist = hist_all[warp];
  const unsigned full = 0xFFFFFFFFu;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const float* src = scores + (size_t)row * ldc;

  uint32_t key[NPL];
  uint32_t alo = 0xFFFFFFFFu, ahi = 0u;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int j = lane + 32 * i;
    key[i] = 0u;
    if (j < n_video) {
      const uint32_t b = __float_as_uint(__ldg(src + j) + 0.0f);
      key[i] = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
      alo = min(alo, key[i]);
      ahi = max(ahi, key[i]);
    }
  }
  alo = __reduce_min_sync(full, alo);
  ahi = __reduce_max_sync(full, ahi);
  int need = k;
  bool ties = false;  // finished with every key of [alo, ahi] equal: take `need` of them by block
  for (int level = 0; level < 5; ++level) {
    if (alo == ahi) {
      ties = true;
      break;
    }
    const uint32_t span = ahi - alo;
    const int shift = span < 256u ? 0 : (32 - __clz((int)span)) - 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0u;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (key[i] >= alo && key[i] <= ahi) atomicAdd(hist + ((key[i] - alo) >> shift), 1u);
    __syncwarp();
    // bin T holding the need-th best: lane l owns bins 255-8l .. 248-8l (descending)
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = hist[255 - 8 * lane - e];
      sum += c[e];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;
    const bool here = excl < (uint32_t)need && (uint32_t)need <= incl;
    const int src_lane = __ffs((int)__ballot_sync(full, here)) - 1;
    uint32_t tbin = 0, greater = 0, in_bin = 0, cum = excl;
    bool found = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (here && !found && cum + c[e] >= (uint32_t)need) {
        found = true;
        tbin = 255 - 8 * lane - e;
        greater = cum;
        in_bin = c[e];
      }
      cum += c[e];
    }
    tbin = __shfl_sync(full, tbin, src_lane);
    greater = __shfl_sync(full, greater, src_lane);
    in_bin = __shfl_sync(full, in_bin, src_lane);
    __syncwarp();  // every lane has read the histogram before the next level clears it
    // keys above bin T are taken; the candidates narrow to bin T
    // (bin T holds a key, so blo <= ahi; no sum below can wrap)
    const uint32_t blo = alo + (tbin << shift);
    ahi = blo + min((1u << shift) - 1u, ahi - blo);
    alo = blo;
    need -= (int)greater;
    if ((uint32_t)need == in_bin) break;  // the whole bin is taken: keys >= alo
  }
  // selected: keys above the range, and, when the range is one tied key,
  // its `need` lowest blocks; else (the whole last bin) every key >= alo
  int32_t* dst = sel + (size_t)row * k;
  int pos = 0, tie_seen = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    bool t;
    if (ties) {
      const bool tie = key[i] == alo;
      const uint32_t tm = __ballot_sync(full, tie);
      t = key[i] > alo || (tie && tie_seen + __popc(tm & lt_mask) < need);
      tie_seen += __popc(tm);
    } else {
      t = key[i] >= alo;
    }
    const uint32_t m = __ballot_sync(full, t);
    const int slot = pos + __popc(m & lt_mask);
    if (t && slot < k) dst[slot] = first_video_block + lane + 32 * i;
    pos += __popc(m);
  }
}

}  // namespace

RouteScratch route_scratch_layout(int H, int d, int n_video) {
  RouteScratch r;
  const size_t split = (size_t)H * n_video * kSplitParts * d * sizeof(uint16_t);
  r.qs = 0;
  r.ks = (split + 255) / 256 * 256;
  r.scores = r.ks + (split + 255) / 256 * 256;
  r.ldc = (n_video + 3) & ~3;
  r.total = r.scores + ((size_t)H * n_video * r.ldc * sizeof(float) + 255) / 256 * 256;
  return r;
}

size_t route_smem_bytes(int d, int n_video) {
  (void)d;
  return sizeof(uint32_t) * (size_t)topk_warp_words(n_video, (n_video + 3) & ~3);
}

cudaError_t launch_route_pipeline(const uint16_t* q, const uint16_t* k, int32_t* kv_sel, int H, int S, int d,
                                  int first_video_block, int n_video, int kk, void* scratch, int* status,
                                  cudaStream_t stream) {
  const RouteScratch r = route_scratch_layout(H, d, n_video);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint16_t* qs = reinterpret_cast<uint16_t*>(base + r.qs);
  uint16_t* ks = reinterpret_cast<uint16_t*>(base + r.ks);
  float* sc = reinterpret_cast<float*>(base + r.scores);
  // 1. pool + split
  const long long warps = 2LL * H * n_video;
  const unsigned pgrid = (unsigned)((warps + 7) / 8);
  if (d == 64)
    pool_split_kernel<64><<<pgrid, 256, 0, stream>>>(q, k, qs, ks, H, S, first_video_block, n_video);
  else
    pool_split_kernel<128><<<pgrid, 256, 0, stream>>>(q, k, qs, ks, H, S, first_video_block, n_video);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. scores on the tensor cores
  CUtensorMap ta, tb;
  if (!encode_bf16_3d(&ta, qs, kSplitParts * d, n_video, H, 64, kGM) ||
      !encode_bf16_3d(&tb, ks, kSplitParts * d, n_video, H, 64, kGN))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int n_tm = (n_video + kGM - 1) / kGM, n_tn = (n_video + kGN - 1) / kGN;
  const long long tiles = (long long)H * n_tm * n_tn;
  if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int ggrid = (int)(tiles < n_sm ? tiles : n_sm);
  CUtensorMap tc;
  if (!encode_f32_3d(&tc, sc, n_video, n_video, H, r.ldc, 32, 32)) return cudaErrorInvalidValue;
  score_gemm_kernel<<<ggrid, kGemmThreads, kGSmem, stream>>>(ta, tb, tc, n_video, kSplitParts * d / 64, n_tm, n_tn,
                                                             (int)tiles,
                                                             status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. top-k per (head, query block): scores in registers up to 2048 video
  // blocks, else staged in shared memory
  const int rows = H * n_video;
  const unsigned rgrid = (unsigned)((rows + 7) / 8);
  if (n_video <= 2048) {
    const int npl = (n_video + 31) / 32;
    if (npl <= 16)
      topk_reg_kernel<16><<<rgrid, 256, 0, stream>>>(sc, kv_sel, rows, n_video, (int)r.ldc, kk, first_video_block);
    else if (npl <= 32)
      topk_reg_kernel<32><<<rgrid, 256, 0, stream>>>(sc, kv_sel, rows, n_video, (int)r.ldc, kk, first_video_block);
    else if (npl <= 48)
      topk_reg_kernel<48><<<rgrid, 256, 0, stream>>>(sc, kv_sel, rows, n_video, (int)r.ldc, kk, first_video_block);
    else
      topk_reg_kernel<64><<<rgrid, 256, 0, stream>>>(sc, kv_sel, rows, n_video, (int)r.ldc, kk, first_video_block);
    return cudaGetLastError();
  }
  const int words = topk_warp_words(n_video, (int)r.ldc);
  int wpc = (int)((200 * 1024) / (words * 4));
  wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
  const size_t tsmem = (size_t)wpc * words * 4;
  e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsmem);
  if (e != cudaSuccess) return e;
  topk_kernel<<<(rows + wpc - 1) / wpc, wpc * 32, tsmem, stream>>>(sc, kv_sel, rows, n_video, (int)r.ldc, kk,
                                                                   first_video_block);
  return cudaGetLastError();
}

}  // namespace h3
