// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace h3 {

constexpr int kSegGuide = 3;
constexpr int kSegOutput = 4;
constexpr int kBlock = 64;
constexpr int kMaxBlocks = 8192;  // S <= 524288: one 16-bit block id, lists fit in shared memory
constexpr int kMaxSmem = 227 * 1024;  // opt-in dynamic shared memory of one CTA on sm_100

// device status word values (the C ABI maps them to H3ATTN_E*)
constexpr int kStatusTimeout = 1;
constexpr int kStatusData = 2;

struct AttnParams {
  int H, S, d;
  int n_blocks, first_video_block, n_video_blocks, k;
  const int32_t* kv_sel;       // [H][nV][k] or null (dense)
  const uint8_t* seg;          // [S]
  const float* times;          // [S]
  const uint4* kv_desc;        // [n_blocks]: see launch_kv_desc
  const float* gtime;          // [n_blocks * 64]: guide key's time, NaN for other keys (read for kind 2)
  const uint32_t* slow_blocks; // [ceil(n_blocks / 32)] bitmap: blocks needing per-key treatment
  // tiles per head: n_dense_tiles of adjacent blocks (2t, 2t+1), then
  // n_paired_tiles read from qpairs[H][n_paired_tiles] (see launch_pair)
  const uint32_t* qpairs;
  int n_dense_tiles, n_paired_tiles;
  // int8 QK (attn kernel instantiated for it): per-token scales of Q and K,
  // [H][scale_stride] with scale_stride = 64 n_blocks (padding rows 0)
  const float* q_scale;
  const float* k_scale;
  int scale_stride;
  uint16_t* o;                 // bf16 [H][S][d]
  float* lse;                  // [H][S] or null
  int* status;                 // device status word
  int pen_on;
  float scale_log2;            // log2(e) / sqrt(d)
  float window, inv_falloff, strength_log2, cap_log2;
  uint32_t wait_polls;         // bounded waits: poll budget
  uint64_t wait_ns;            // bounded waits: time budget
};

int attn_smem_bytes(int d, int n_blocks, bool qk8 = false);
// qk8: tq / tk map int8 Q / K codes ({d, S, H} bytes, box {d, 64}) and the QK
// products run as int8 MMAs (d = 128 only)
cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnParams& p, int n_ctas, cudaStream_t stream, bool qk8 = false);

// per-token int8 quantisation of Q and K (quant.cu): codes [H][S][d], scales
// [H][stride] (rows S..stride-1 get 0)
cudaError_t launch_quant_qk(const uint16_t* q, const uint16_t* k, int8_t* q8, int8_t* k8, float* sq, float* sk,
                            int H, int S, int d, int stride, cudaStream_t stream);

// float32 tensor [dim2][dim1][pitch] (dim0 <= pitch valid columns, pitch a
// multiple of 4) as a 3-D TMA map with a {box0, box1, 1} box and 128-byte
// swizzle (box0 = 32)
bool encode_f32_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint64_t pitch,
                   uint32_t box0, uint32_t box1);

// int8 tensor [dim2][dim1][dim0] as a 3-D TMA map with a {box0, box1, 1} box
// and 128-byte swizzle (box0 <= 128)
bool encode_u8_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                  uint32_t box1);

// kv_desc[b] for every key block b, over its valid rows (n of them):
//   x = n | kind << 8 | split << 16, y / z = time bits of runs a / b
//   kind 0: no guide row;
//   kind 1: rows [0, split) and [split, n) each all guide rows of one time
//           (y, z) or all other rows (time NaN); split = n for a single run;
//   kind 2: anything else (per-row times needed).
// And, when times is not null, gtime[r] for every row r < 64 n_blocks: the
// row's time if it is a guide row below S, NaN otherwise.
// slow[b / 32] bit b % 32: block b needs per-key treatment in the attention
// kernel (fewer than 64 valid rows, kind 2, or a kind-1 split inside a
// 16-key group), for every block b < 32 ceil(n_blocks / 32).
cudaError_t launch_kv_desc(const uint8_t* seg, const float* times, int S, int n_blocks, uint4* kv_desc,
                           float* gtime, uint32_t* slow, cudaStream_t stream);

// Query-block pairing (pair.cu).  With routing, the attention tiles of a head
// are the adjacent pairs (2t, 2t+1) of blocks below paired_first_block(fvb)
// (the dense prefix, rounded up to an even block), then paired_tiles(...)
// tiles of blocks from that point on, paired within groups of kPairGroup
// consecutive blocks by routed-list overlap.  Entry: block a | block b << 16,
// b = kNoPair for a tile holding block a alone.
constexpr int kPairGroup = 32;
constexpr uint32_t kNoPair = 0xFFFFu;
inline int paired_first_block(int first_video_block) { return (first_video_block + 1) & ~1; }
inline int paired_tiles(int n_blocks, int first_video_block) {
  const int n = n_blocks - paired_first_block(first_video_block);
  return n <= 0 ? 0 : n / kPairGroup * (kPairGroup / 2) + (n % kPairGroup + 1) / 2;
}
// pairs[H][paired_tiles(n_blocks, first_video_block)] from kv_sel[H][nV][k]
cudaError_t launch_pair(const int32_t* kv_sel, int H, int n_blocks, int first_video_block, int k,
                        uint32_t* pairs, cudaStream_t stream);

// mean-pool blocks [first_block, first_block + n_out) of up to two bf16 [H][S][d] tensors
cudaError_t launch_pool(const uint16_t* x0, float* out0, const uint16_t* x1, float* out1, int H, int S,
                        int d, int first_block, int n_out, cudaStream_t stream);

// bf16 tensor [dim2][dim1][dim0] (dim0 contiguous) as a 3-D TMA map with a
// {box0, box1, 1} box and 128-byte swizzle; out-of-range elements read as zero
bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                    uint32_t box1);

// Routing scratch (byte offsets): the pooled centroids of Q and K as three
// bf16 parts, [H][n_video][kSplitParts d], and the fp32 score matrix
// [H][n_video][ldc].
constexpr int kSplitParts = 6;
struct RouteScratch {
  size_t qs, ks, scores, ldc, total;
};
RouteScratch route_scratch_layout(int H, int d, int n_video);
size_t route_smem_bytes(int d, int n_video);  // shared memory of one top-k warp

// pool + split, tensor-core pooled scores, top-k: kv_sel[H][n_video][k]
cudaError_t launch_route_pipeline(const uint16_t* q, const uint16_t* k, int32_t* kv_sel, int H, int S, int d,
                                  int first_video_block, int n_video, int kk, void* scratch, int* status,
                                  cudaStream_t stream);

// pooled tail term (h3attn_tail_correct): scratch byte offsets of the bf16
// weights [H][n_video][ldk], the transposed pooled V [H][d][ldk], the tail
// outputs [H][n_video][d] (bf16) and the per-block log mass and 1 / mass
struct TailScratch {
  size_t w, vpt, ot, lt, inv_sum, total, ldk;
};
TailScratch tail_scratch_layout(int H, int d, int n_video);
// scores: the fp32 pooled scores [H][n_video][ldc] routing left; o / lse
// updated in place for the rows of video query blocks
cudaError_t launch_tail(const uint16_t* v, const float* scores, size_t ldc, const int32_t* kv_sel, int kk, int H,
                        int S, int d, int first_block, int n_video, uint16_t* o, float* lse, void* scratch,
                        int* status, cudaStream_t stream);

// partition merge (h3attn_merge): up to kMaxMergeParts partitions, passed by value
constexpr int kMaxMergeParts = 8;
struct MergeParts {
  const uint16_t* o[kMaxMergeParts];  // bf16 [rows][d]
  const float* lse[kMaxMergeParts];   // [rows]
  float log_w[kMaxMergeParts];
  int n;
};
cudaError_t launch_merge(const MergeParts& parts, long long rows, int d, uint16_t* o, float* lse,
                         cudaStream_t stream);

cudaError_t launch_selftest_timeout(int* status, uint32_t polls, cudaStream_t stream);

}  // namespace h3
