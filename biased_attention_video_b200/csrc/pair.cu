// Query-block pairing for the attention kernel's 128-row tiles.
//
// A tile of the attention kernel holds two 64-row query blocks and walks the
// union of their key-block lists ("H3 SLA Attention", "How it works": every
// video query block attends its own routed blocks plus the forced ones); a key
// block that only one of the two attends still costs the whole tile's S and PV
// products.  Pairing the query blocks whose routed lists overlap most shrinks
// the unions.  Which blocks share a tile never changes a result: every row
// still attends exactly its own blocks, the others are masked.
//
// Video query blocks [first_paired, n_blocks) are cut into groups of 32
// consecutive blocks (the last group may be shorter).  Within a group the
// matching is greedy: repeatedly take the pair of unmatched blocks with the
// largest overlap |list_a & list_b| (ties to the lower block indices) until
// fewer than two are left; an odd block out gets a tile of its own.  One warp
// handles one (group, head): lane i owns block i's list as a bitmap over the
// video key blocks, the 32 x 32 overlaps are popcounts of bitmap words passed
// around the warp by shuffles, and every round of the greedy matching is one
// warp-wide max.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace h3 {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// grid (n_groups, H), 32 threads; dynamic shared memory: 32 bitmaps of
// `stride` words (stride odd, so that lane a reading word w of its own bitmap
// hits bank (a * stride + w) % 32, all distinct).
__global__ void __launch_bounds__(32) pair_kernel(const int32_t* __restrict__ kv_sel, int n_blocks,
                                                   int first_video_block, int n_video, int k, int first_paired,
                                                   int n_paired_tiles, int words, int stride,
                                                   uint32_t* __restrict__ pairs) {
  extern __shared__ uint32_t bm[];
  const int lane = threadIdx.x;
  const int g = blockIdx.x, head = blockIdx.y;
  const int b0 = first_paired + g * kPairGroup;  // first query block of the group
  const int gs = min(kPairGroup, n_blocks - b0);  // blocks in this group

  for (int i = lane; i < kPairGroup * stride; i += 32) bm[i] = 0u;
  __syncwarp();
  // lists -> bitmaps over video key blocks (entries outside the video range
  // are skipped here; the attention kernel flags them)
  for (int i = 0; i < gs; ++i) {
    const int32_t* lst = kv_sel + ((size_t)head * n_video + (b0 + i - first_video_block)) * k;
    for (int e = lane; e < k; e += 32) {
      const int v = __ldg(lst + e) - first_video_block;
      if (v >= 0 && v < n_video) atomicOr(bm + i * stride + (v >> 5), 1u << (v & 31));
    }
  }
  __syncwarp();

  // ov[b] = |list_lane & list_b|
  uint32_t ov[kPairGroup];
#pragma unroll
  for (int b = 0; b < kPairGroup; ++b) ov[b] = 0u;
  for (int w = 0; w < words; ++w) {
    const uint32_t x = bm[lane * stride + w];
#pragma unroll
    for (int b = 0; b < kPairGroup; ++b) ov[b] += __popc(x & __shfl_sync(kFull, x, b));
  }

  // greedy matching; key = overlap << 10 | (31 - lower) << 5 | (31 - higher),
  // so the warp max picks the largest overlap, then the lowest pair
  uint32_t matched = gs >= 32 ? 0u : ~((1u << gs) - 1u);
  uint32_t* out = pairs + (size_t)head * n_paired_tiles + (size_t)g * (kPairGroup / 2);
  int t = 0;
  while (__popc(~matched) >= 2) {
    uint32_t best = 0u;
    if (!((matched >> lane) & 1u)) {
#pragma unroll
      for (int b = 0; b < kPairGroup; ++b) {
        if (b == lane || ((matched >> b) & 1u)) continue;
        const uint32_t lo = (uint32_t)min(lane, b), hi = (uint32_t)max(lane, b);
        const uint32_t key = (ov[b] << 10) | ((31u - lo) << 5) | (31u - hi);
        best = max(best, key);
      }
    }
    best = __reduce_max_sync(kFull, best);
    const int a = 31 - (int)((best >> 5) & 31u), b = 31 - (int)(best & 31u);
    matched |= (1u << a) | (1u << b);
    if (lane == 0) out[t] = (uint32_t)(b0 + a) | ((uint32_t)(b0 + b) << 16);
    ++t;
  }
  if (~matched != 0u && lane == 0) out[t] = (uint32_t)(b0 + __ffs((int)~matched) - 1) | (kNoPair << 16);
}

}  // namespace

cudaError_t launch_pair(const int32_t* kv_sel, int H, int n_blocks, int first_video_block, int k,
                        uint32_t* pairs, cudaStream_t stream) {
  const int first_paired = paired_first_block(first_video_block);
  const int n_paired = n_blocks - first_paired;
  if (n_paired <= 0) return cudaSuccess;
  const int n_video = n_blocks - first_video_block;
  const int words = (n_video + 31) / 32;
  const int stride = words | 1;
  // at most 32 x 257 words (n_video <= kMaxBlocks): under the default 48 KB
  const size_t smem = (size_t)kPairGroup * stride * sizeof(uint32_t);
  const dim3 grid((unsigned)((n_paired + kPairGroup - 1) / kPairGroup), (unsigned)H);
  pair_kernel<<<grid, 32, smem, stream>>>(kv_sel, n_blocks, first_video_block, n_video, k, first_paired,
                                          paired_tiles(n_blocks, first_video_block), words, stride, pairs);
  return cudaGetLastError();
}

}  // namespace h3
