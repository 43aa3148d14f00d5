#include <algorithm>
// C ABI of libh3attn: argument validation, block plan, workspace layout,
// TMA descriptors and kernel launches.  See include/h3attn.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <atomic>
#include <new>
#include <cstdint>
#include <cstring>

#include "h3attn.h"
#include "kernels.cuh"


namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;
constexpr uint32_t kWaitPolls = 0xFFFFFFFFu;  // no poll bound: only the time bound applies
// poll bound of the attention kernels' waits for the calls launched next
// (h3attn_set_wait_polls; 0 = kWaitPolls)
std::atomic<uint32_t> g_wait_polls{0u};
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait: far above any legitimate stall
using h3::kMaxSmem;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct WsLayout {
  size_t desc, gtime, slow, pairs, route, total;
};

// Attention scratch after the status word: per-key-block descriptors, per-key
// guide times (a guide key's time, NaN for every other key; padded to whole
// blocks), and the bitmap of key blocks that need per-key treatment.
size_t attn_scratch_bytes(int n_blocks) {
  return align_up((size_t)n_blocks * sizeof(uint4)) + align_up((size_t)n_blocks * h3::kBlock * sizeof(float)) +
         align_up((size_t)(n_blocks + 31) / 32 * sizeof(uint32_t));
}

// query-block pair table of a routed call: one word per paired tile and head
size_t pair_bytes(const h3attn_plan* plan) {
  return plan->n_video_blocks > 0
             ? align_up((size_t)plan->H * h3::paired_tiles(plan->n_blocks, plan->first_video_block) * sizeof(uint32_t))
             : 0;
}

// status word | per-key-block descriptors | per-key guide times | slow-block
// bitmap | query-block pairs | routing scratch
WsLayout ws_layout(const h3attn_plan* plan) {
  WsLayout w;
  w.desc = kStatusBytes;
  w.gtime = w.desc + align_up((size_t)plan->n_blocks * sizeof(uint4));
  w.slow = w.gtime + align_up((size_t)plan->n_blocks * h3::kBlock * sizeof(float));
  w.pairs = kStatusBytes + attn_scratch_bytes(plan->n_blocks);
  w.route = w.pairs + pair_bytes(plan);
  w.total = w.route +
            (plan->n_video_blocks > 0 ? h3::route_scratch_layout(plan->H, plan->d, plan->n_video_blocks).total : 0);
  return w;
}

bool plan_ok(const h3attn_plan* p) {
  return p != nullptr && p->H > 0 && p->S > 0 && (p->d == 64 || p->d == 128) && p->block == h3::kBlock &&
         p->n_blocks == (p->S + p->block - 1) / p->block && p->n_blocks <= h3::kMaxBlocks &&
         p->first_video_block >= 0 && p->first_video_block <= p->n_blocks &&
         p->n_video_blocks == p->n_blocks - p->first_video_block && p->n_forced == p->first_video_block &&
         (p->n_video_blocks == 0 || (p->k >= 1 && p->k <= p->n_video_blocks));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 [H][S][d] viewed as 3-D {d, S, H}; box {64, 64, 1}
bool make_map(CUtensorMap* m, const void* base, int H, int S, int d) {
  return h3::encode_bf16_3d(m, base, (uint64_t)d, (uint64_t)S, (uint64_t)H, 64, 64);
}

bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.0f; }

// int8 QK scratch: codes of Q and K [H][S][d], then their per-token scales
// [H][64 n_blocks] (a whole-block stride keeps each head's scales 16-byte
// aligned; padding rows hold 0)
struct Qk8Layout {
  size_t q8, k8, sq, sk, total;
  int stride;
};
Qk8Layout qk8_layout(const h3attn_plan* plan) {
  Qk8Layout l;
  l.stride = plan->n_blocks * h3::kBlock;
  const size_t codes = (size_t)plan->H * plan->S * plan->d;
  const size_t scales = (size_t)plan->H * l.stride * sizeof(float);
  l.q8 = 0;
  l.k8 = align_up(codes);
  l.sq = l.k8 + align_up(codes);
  l.sk = l.sq + align_up(scales);
  l.total = l.sk + align_up(scales);
  return l;
}

struct Qk8Operands {
  const int8_t *q8, *k8;
  const float *sq, *sk;
  int stride;
};

// qk8: int8 Q / K codes and scales (q, k unused then), or null for bf16 Q / K
int forward_impl(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const uint8_t* seg, const float* times, const h3attn_penalty* pen, const int32_t* kv_sel,
                 uint16_t* o, float* lse, void* ws, size_t ws_bytes, size_t ws_needed, cudaStream_t stream,
                 const Qk8Operands* qk8 = nullptr) {
  if (!plan_ok(plan)) return H3ATTN_EINVAL;
  if (qk8 == nullptr && (!q || !k)) return H3ATTN_EINVAL;
  if (!v || !seg || !o) return H3ATTN_EINVAL;
  if (ws == nullptr || ws_bytes < ws_needed) return H3ATTN_EWORKSPACE;
  if ((qk8 == nullptr && (!aligned16(q) || !aligned16(k))) || !aligned16(v) || !aligned16(o) || !aligned16(ws))
    return H3ATTN_EALIGN;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return H3ATTN_EALIGN;
  bool pen_on = false;
  if (pen != nullptr) {
    if (!finite_nonneg(pen->strength) || !finite_nonneg(pen->window) || !finite_nonneg(pen->cap) ||
        !std::isfinite(pen->falloff))
      return H3ATTN_EINVAL;
    pen_on = pen->strength > 0.0f && pen->cap > 0.0f;
    if (pen_on && !(pen->falloff > 0.0f)) return H3ATTN_EINVAL;
    if (pen_on && times == nullptr) return H3ATTN_EINVAL;
    if (pen_on && (reinterpret_cast<uintptr_t>(times) & 3u)) return H3ATTN_EALIGN;
  }
  if (h3::attn_smem_bytes(plan->d, plan->n_blocks, qk8 != nullptr) > kMaxSmem) return H3ATTN_EUNSUPPORTED;
  const bool routed = kv_sel != nullptr && plan->n_video_blocks > 0;

  h3::AttnParams p{};
  p.H = plan->H;
  p.S = plan->S;
  p.d = plan->d;
  p.n_blocks = plan->n_blocks;
  p.first_video_block = plan->first_video_block;
  p.n_video_blocks = plan->n_video_blocks;
  p.k = plan->k;
  p.kv_sel = routed ? kv_sel : nullptr;
  p.seg = seg;
  p.times = times;
  p.o = o;
  p.lse = lse;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.status = reinterpret_cast<int*>(wsb);
  const WsLayout wl = ws_layout(plan);
  p.kv_desc = reinterpret_cast<const uint4*>(wsb + wl.desc);
  p.gtime = reinterpret_cast<const float*>(wsb + wl.gtime);
  p.slow_blocks = reinterpret_cast<const uint32_t*>(wsb + wl.slow);
  p.pen_on = pen_on ? 1 : 0;
  const float log2e = 1.4426950408889634f;
  p.scale_log2 = log2e / std::sqrt((float)plan->d);
  if (pen_on) {
    p.window = pen->window;
    p.inv_falloff = 1.0f / pen->falloff;
    p.strength_log2 = pen->strength * log2e;
    p.cap_log2 = pen->cap * log2e;
  }
  const uint32_t polls = g_wait_polls.load(std::memory_order_relaxed);
  p.wait_polls = polls == 0u ? kWaitPolls : polls;
  p.wait_ns = kWaitNs;
  // routed: adjacent pairs over the dense prefix, then the overlap pairing
  p.qpairs = routed ? reinterpret_cast<const uint32_t*>(wsb + wl.pairs) : nullptr;
  p.n_dense_tiles = routed ? h3::paired_first_block(plan->first_video_block) / 2 : (plan->n_blocks + 1) / 2;
  p.n_paired_tiles = routed ? h3::paired_tiles(plan->n_blocks, plan->first_video_block) : 0;
  const int n_qtiles = p.n_dense_tiles + p.n_paired_tiles;

  CUtensorMap tq, tk, tv;
  if (qk8 != nullptr) {
    p.q_scale = qk8->sq;
    p.k_scale = qk8->sk;
    p.scale_stride = qk8->stride;
    if (!h3::encode_u8_3d(&tq, qk8->q8, (uint64_t)plan->d, (uint64_t)plan->S, (uint64_t)plan->H, 128, 64) ||
        !h3::encode_u8_3d(&tk, qk8->k8, (uint64_t)plan->d, (uint64_t)plan->S, (uint64_t)plan->H, 128, 64))
      return H3ATTN_ECUDA;
  } else if (!make_map(&tq, q, plan->H, plan->S, plan->d) || !make_map(&tk, k, plan->H, plan->S, plan->d)) {
    return H3ATTN_ECUDA;
  }
  if (!make_map(&tv, v, plan->H, plan->S, plan->d)) return H3ATTN_ECUDA;
  if (h3::launch_kv_desc(seg, pen_on ? times : nullptr, plan->S, plan->n_blocks,
                         reinterpret_cast<uint4*>(wsb + wl.desc), reinterpret_cast<float*>(wsb + wl.gtime),
                         reinterpret_cast<uint32_t*>(wsb + wl.slow), stream) != cudaSuccess)
    return H3ATTN_ECUDA;
  if (routed && h3::launch_pair(kv_sel, plan->H, plan->n_blocks, plan->first_video_block, plan->k,
                                reinterpret_cast<uint32_t*>(wsb + wl.pairs), stream) != cudaSuccess)
    return H3ATTN_ECUDA;
  if (h3::launch_attn(tq, tk, tv, p, n_qtiles * plan->H, stream, qk8 != nullptr) != cudaSuccess) return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

}  // namespace

namespace h3 {
bool encode_u8_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                  uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0, dim0 * dim1};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_f32_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint64_t pitch,
                   uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {pitch * 4, pitch * dim1 * 4};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                    uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace h3

extern "C" {

int h3attn_plan_init(h3attn_plan* plan, int H, int S, int d, int block, double sparsity, const uint8_t* seg_host) {
  if (plan == nullptr || seg_host == nullptr || H <= 0 || S <= 0) return H3ATTN_EINVAL;
  if (!(sparsity >= 0.0 && sparsity < 1.0)) return H3ATTN_EINVAL;
  if (!(d == 64 || d == 128) || block != h3::kBlock) return H3ATTN_EUNSUPPORTED;
  const int n_blocks = (S + block - 1) / block;
  if (n_blocks > h3::kMaxBlocks) return H3ATTN_EUNSUPPORTED;
  int prefix = 0;
  while (prefix < S && seg_host[prefix] != H3ATTN_SEG_GUIDE && seg_host[prefix] != H3ATTN_SEG_OUTPUT) ++prefix;
  for (int r = prefix; r < S; ++r)
    if (seg_host[r] != H3ATTN_SEG_GUIDE && seg_host[r] != H3ATTN_SEG_OUTPUT) return H3ATTN_EUNSUPPORTED;
  for (int r = 0; r < S; ++r)
    if (seg_host[r] > H3ATTN_SEG_OUTPUT) return H3ATTN_EINVAL;
  h3attn_plan p{};
  p.H = H;
  p.S = S;
  p.d = d;
  p.block = block;
  p.sparsity = sparsity;
  p.n_blocks = n_blocks;
  p.prefix_rows = prefix;
  p.first_video_block = (prefix + block - 1) / block;
  p.n_forced = p.first_video_block;
  p.n_video_blocks = n_blocks - p.first_video_block;
  if (p.n_video_blocks > 0) {
    const double want = std::ceil((1.0 - sparsity) * (double)p.n_video_blocks - 1e-9);
    int kk = (int)want;
    if (kk < 1) kk = 1;
    if (kk > p.n_video_blocks) kk = p.n_video_blocks;
    p.k = kk;
  } else {
    p.k = 0;
  }
  *plan = p;
  return H3ATTN_OK;
}

size_t h3attn_workspace_bytes(const h3attn_plan* plan) {
  if (!plan_ok(plan)) return 0;
  return ws_layout(plan).total;
}

int h3attn_pool(const h3attn_plan* plan, const uint16_t* x, int first_block, int n_out, float* out, void* stream) {
  if (!plan_ok(plan) || x == nullptr || out == nullptr) return H3ATTN_EINVAL;
  if (first_block < 0 || n_out < 0 || first_block + n_out > plan->n_blocks) return H3ATTN_EINVAL;
  if (!aligned16(x) || !aligned16(out)) return H3ATTN_EALIGN;
  if (n_out == 0) return H3ATTN_OK;
  if (h3::launch_pool(x, out, nullptr, nullptr, plan->H, plan->S, plan->d, first_block, n_out,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

int h3attn_route(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, int32_t* kv_sel, void* ws,
                 size_t ws_bytes, void* stream) {
  if (!plan_ok(plan) || q == nullptr || k == nullptr || kv_sel == nullptr) return H3ATTN_EINVAL;
  if (plan->n_video_blocks == 0) return H3ATTN_EINVAL;
  const WsLayout w = ws_layout(plan);
  if (ws == nullptr || ws_bytes < w.total) return H3ATTN_EWORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(kv_sel) & 3u))
    return H3ATTN_EALIGN;
  if (h3::route_smem_bytes(plan->d, plan->n_video_blocks) > (size_t)kMaxSmem) return H3ATTN_EUNSUPPORTED;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  if (h3::launch_route_pipeline(q, k, kv_sel, plan->H, plan->S, plan->d, plan->first_video_block,
                                plan->n_video_blocks, plan->k, wsb + w.route, reinterpret_cast<int*>(wsb),
                                static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

int h3attn_forward(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint8_t* seg, const float* times, const h3attn_penalty* pen, const int32_t* kv_sel,
                   uint16_t* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!plan_ok(plan)) return H3ATTN_EINVAL;
  // a routed call also needs the query-block pair table
  const size_t need = kStatusBytes + attn_scratch_bytes(plan->n_blocks) + (kv_sel != nullptr ? pair_bytes(plan) : 0);
  if (kv_sel != nullptr && (reinterpret_cast<uintptr_t>(kv_sel) & 3u)) return H3ATTN_EALIGN;
  return forward_impl(plan, q, k, v, seg, times, pen, kv_sel, o, lse, ws, ws_bytes, need,
                      static_cast<cudaStream_t>(stream));
}

int h3attn_attend_host(const h3attn_plan* plan, const uint16_t* q_host, const uint16_t* k_host,
                       const uint16_t* v_host, const uint8_t* seg_host, const float* times_host,
                       const h3attn_penalty* pen, uint16_t* o_host, float* lse_host, uint16_t* q, uint16_t* k,
                       uint16_t* v, uint8_t* seg, float* times, int32_t* kv_sel, uint16_t* o, float* lse, void* ws,
                       size_t ws_bytes, int chunk_heads, void* stream, void* copy_in_stream,
                       void* copy_out_stream) {
  if (!plan_ok(plan)) return H3ATTN_EINVAL;
  if (!q_host || !k_host || !v_host || !seg_host || !o_host || !q || !k || !v || !seg || !o) return H3ATTN_EINVAL;
  const bool routed = plan->n_video_blocks > 0 && plan->k < plan->n_video_blocks;
  if (routed && kv_sel == nullptr) return H3ATTN_EINVAL;
  if ((lse_host == nullptr) != (lse == nullptr)) return H3ATTN_EINVAL;
  if (pen != nullptr && (times_host == nullptr || times == nullptr)) return H3ATTN_EINVAL;
  if (chunk_heads < 1 || chunk_heads > plan->H) return H3ATTN_EINVAL;
  if (ws == nullptr || ws_bytes < h3attn_workspace_bytes(plan)) return H3ATTN_EWORKSPACE;
  const cudaStream_t sc = static_cast<cudaStream_t>(stream);
  const cudaStream_t si = static_cast<cudaStream_t>(copy_in_stream);
  const cudaStream_t so = static_cast<cudaStream_t>(copy_out_stream);
  const size_t per_head = (size_t)plan->S * plan->d;  // elements of one head of Q/K/V/O
  const size_t sel_per_head = (size_t)plan->n_video_blocks * plan->k;
  const int n_chunks = (plan->H + chunk_heads - 1) / chunk_heads;
  // two events per chunk (inputs landed, outputs ready), one for the end and
  // one for the start
  const int n_events = 2 * n_chunks + 2;
  cudaEvent_t* evs = new (std::nothrow) cudaEvent_t[n_events];
  if (evs == nullptr) return H3ATTN_ECUDA;
  int n_ev = 0, rc = H3ATTN_OK;
  for (; n_ev < n_events; ++n_ev)
    if (cudaEventCreateWithFlags(&evs[n_ev], cudaEventDisableTiming) != cudaSuccess) {
      rc = H3ATTN_ECUDA;
      break;
    }
  auto copy = [&](void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t st) {
    if (rc == H3ATTN_OK && cudaMemcpyAsync(dst, src, bytes, kind, st) != cudaSuccess) rc = H3ATTN_ECUDA;
  };
  auto record = [&](cudaEvent_t e, cudaStream_t st) {
    if (rc == H3ATTN_OK && cudaEventRecord(e, st) != cudaSuccess) rc = H3ATTN_ECUDA;
  };
  auto wait = [&](cudaStream_t st, cudaEvent_t e) {
    if (rc == H3ATTN_OK && cudaStreamWaitEvent(st, e, 0) != cudaSuccess) rc = H3ATTN_ECUDA;
  };
  // the copies start once `stream` has reached this call: work queued there
  // before (an earlier call still reading or writing these buffers) is done
  record(evs[2 * n_chunks + 1], sc);
  wait(si, evs[2 * n_chunks + 1]);
  wait(so, evs[2 * n_chunks + 1]);
  // the per-sequence inputs go first, with the first chunk
  copy(seg, seg_host, (size_t)plan->S, cudaMemcpyHostToDevice, si);
  if (times_host != nullptr && times != nullptr)
    copy(times, times_host, (size_t)plan->S * sizeof(float), cudaMemcpyHostToDevice, si);
  for (int c = 0; c < n_chunks && rc == H3ATTN_OK; ++c) {
    const int h0 = c * chunk_heads, hc = std::min(chunk_heads, plan->H - h0);
    const size_t off = (size_t)h0 * per_head, bytes = (size_t)hc * per_head * sizeof(uint16_t);
    copy(q + off, q_host + off, bytes, cudaMemcpyHostToDevice, si);
    copy(k + off, k_host + off, bytes, cudaMemcpyHostToDevice, si);
    copy(v + off, v_host + off, bytes, cudaMemcpyHostToDevice, si);
    record(evs[2 * c], si);
    wait(sc, evs[2 * c]);
    if (rc != H3ATTN_OK) break;
    h3attn_plan cp = *plan;  // the same sequence, hc heads
    cp.H = hc;
    int32_t* sel = routed ? kv_sel + (size_t)h0 * sel_per_head : nullptr;
    if (routed) {
      rc = h3attn_route(&cp, q + off, k + off, sel, ws, ws_bytes, stream);
      if (rc != H3ATTN_OK) break;
    }
    rc = h3attn_forward(&cp, q + off, k + off, v + off, seg, times, pen, sel, o + off,
                        lse != nullptr ? lse + (size_t)h0 * plan->S : nullptr, ws, ws_bytes, stream);
    if (rc != H3ATTN_OK) break;
    record(evs[2 * c + 1], sc);
    wait(so, evs[2 * c + 1]);
    copy(o_host + off, o + off, bytes, cudaMemcpyDeviceToHost, so);
    if (lse != nullptr)
      copy(lse_host + (size_t)h0 * plan->S, lse + (size_t)h0 * plan->S, (size_t)hc * plan->S * sizeof(float),
           cudaMemcpyDeviceToHost, so);
  }
  // the caller's stream completes after the last copy back
  record(evs[2 * n_chunks], so);
  wait(sc, evs[2 * n_chunks]);
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(evs[i]);  // released once their work is done
  delete[] evs;
  return rc;
}

int h3attn_merge(int n_parts, const uint16_t* const* o_parts, const float* const* lse_parts, const float* log_w,
                 int H, int S, int d, uint16_t* o, float* lse, void* stream) {
  if (n_parts < 1 || n_parts > h3::kMaxMergeParts || o_parts == nullptr || lse_parts == nullptr || o == nullptr)
    return H3ATTN_EINVAL;
  if (H <= 0 || S <= 0) return H3ATTN_EINVAL;
  if (!(d == 64 || d == 128)) return H3ATTN_EUNSUPPORTED;
  h3::MergeParts parts{};
  parts.n = n_parts;
  for (int i = 0; i < n_parts; ++i) {
    if (o_parts[i] == nullptr || lse_parts[i] == nullptr) return H3ATTN_EINVAL;
    if ((reinterpret_cast<uintptr_t>(o_parts[i]) & 15u) || (reinterpret_cast<uintptr_t>(lse_parts[i]) & 3u))
      return H3ATTN_EALIGN;
    const float lw = log_w != nullptr ? log_w[i] : 0.0f;
    if (std::isnan(lw) || lw == INFINITY) return H3ATTN_EINVAL;
    parts.o[i] = o_parts[i];
    parts.lse[i] = lse_parts[i];
    parts.log_w[i] = lw;
  }
  if ((reinterpret_cast<uintptr_t>(o) & 15u) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return H3ATTN_EALIGN;
  if (h3::launch_merge(parts, (long long)H * S, d, o, lse, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

size_t h3attn_tail_workspace_bytes(const h3attn_plan* plan) {
  if (!plan_ok(plan) || plan->n_video_blocks == 0) return 0;
  return h3::tail_scratch_layout(plan->H, plan->d, plan->n_video_blocks).total;
}

int h3attn_tail_correct(const h3attn_plan* plan, const uint16_t* v, const int32_t* kv_sel, uint16_t* o, float* lse,
                        void* ws, size_t ws_bytes, void* tail_ws, size_t tail_ws_bytes, void* stream) {
  if (!plan_ok(plan) || plan->n_video_blocks == 0) return H3ATTN_EINVAL;
  if (v == nullptr || kv_sel == nullptr || o == nullptr || lse == nullptr) return H3ATTN_EINVAL;
  const WsLayout w = ws_layout(plan);
  if (ws == nullptr || ws_bytes < w.total) return H3ATTN_EWORKSPACE;
  if (tail_ws == nullptr || tail_ws_bytes < h3attn_tail_workspace_bytes(plan)) return H3ATTN_EWORKSPACE;
  if (!aligned16(v) || !aligned16(o) || !aligned16(tail_ws) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(kv_sel) & 3u))
    return H3ATTN_EALIGN;
  const size_t bitmap_smem = (size_t)8 * ((plan->n_video_blocks + 31) / 32) * 4;
  if (bitmap_smem > (size_t)kMaxSmem) return H3ATTN_EUNSUPPORTED;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const h3::RouteScratch r = h3::route_scratch_layout(plan->H, plan->d, plan->n_video_blocks);
  const float* scores = reinterpret_cast<const float*>(wsb + w.route + r.scores);
  if (h3::launch_tail(v, scores, r.ldc, kv_sel, plan->k, plan->H, plan->S, plan->d, plan->first_video_block,
                      plan->n_video_blocks, o, lse, tail_ws, reinterpret_cast<int*>(wsb),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

size_t h3attn_qk8_workspace_bytes(const h3attn_plan* plan) {
  if (!plan_ok(plan)) return 0;
  return qk8_layout(plan).total;
}

int h3attn_quantize_qk(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, void* qk8_ws,
                       size_t qk8_ws_bytes, void* stream) {
  if (!plan_ok(plan) || q == nullptr || k == nullptr) return H3ATTN_EINVAL;
  const Qk8Layout l = qk8_layout(plan);
  if (qk8_ws == nullptr || qk8_ws_bytes < l.total) return H3ATTN_EWORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(qk8_ws)) return H3ATTN_EALIGN;
  uint8_t* b = static_cast<uint8_t*>(qk8_ws);
  if (h3::launch_quant_qk(q, k, reinterpret_cast<int8_t*>(b + l.q8), reinterpret_cast<int8_t*>(b + l.k8),
                          reinterpret_cast<float*>(b + l.sq), reinterpret_cast<float*>(b + l.sk), plan->H, plan->S,
                          plan->d, l.stride, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

int h3attn_forward_qk8(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const uint8_t* seg, const float* times, const h3attn_penalty* pen, const int32_t* kv_sel,
                       uint16_t* o, float* lse, void* ws, size_t ws_bytes, void* qk8_ws, size_t qk8_ws_bytes,
                       void* stream) {
  if (!plan_ok(plan)) return H3ATTN_EINVAL;
  if (plan->d != 128) return H3ATTN_EUNSUPPORTED;
  if (kv_sel != nullptr && (reinterpret_cast<uintptr_t>(kv_sel) & 3u)) return H3ATTN_EALIGN;
  const int rc = h3attn_quantize_qk(plan, q, k, qk8_ws, qk8_ws_bytes, stream);
  if (rc != H3ATTN_OK) return rc;
  const Qk8Layout l = qk8_layout(plan);
  const uint8_t* b = static_cast<const uint8_t*>(qk8_ws);
  const Qk8Operands ops{reinterpret_cast<const int8_t*>(b + l.q8), reinterpret_cast<const int8_t*>(b + l.k8),
                        reinterpret_cast<const float*>(b + l.sq), reinterpret_cast<const float*>(b + l.sk), l.stride};
  const size_t need = kStatusBytes + attn_scratch_bytes(plan->n_blocks) + (kv_sel != nullptr ? pair_bytes(plan) : 0);
  return forward_impl(plan, q, k, v, seg, times, pen, kv_sel, o, lse, ws, ws_bytes, need,
                      static_cast<cudaStream_t>(stream), &ops);
}

size_t h3attn_dense_workspace_bytes(int S) {
  if (S <= 0) return 0;
  const int n_blocks = (S + h3::kBlock - 1) / h3::kBlock;
  return kStatusBytes + attn_scratch_bytes(n_blocks);
}

int h3attn_dense_biased(int H, int S, int d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint8_t* seg, const float* times, const h3attn_penalty* pen, uint16_t* o, float* lse,
                        void* ws, size_t ws_bytes, void* stream) {
  if (H <= 0 || S <= 0) return H3ATTN_EINVAL;
  if (!(d == 64 || d == 128)) return H3ATTN_EUNSUPPORTED;
  h3attn_plan p{};
  p.H = H;
  p.S = S;
  p.d = d;
  p.block = h3::kBlock;
  p.sparsity = 0.0;
  p.n_blocks = (S + h3::kBlock - 1) / h3::kBlock;
  if (p.n_blocks > h3::kMaxBlocks) return H3ATTN_EUNSUPPORTED;
  p.prefix_rows = S;
  p.first_video_block = p.n_blocks;
  p.n_forced = p.n_blocks;
  p.n_video_blocks = 0;
  p.k = 0;
  return forward_impl(&p, q, k, v, seg, times, pen, nullptr, o, lse, ws, ws_bytes, h3attn_dense_workspace_bytes(S),
                      static_cast<cudaStream_t>(stream));
}

int h3attn_check(void* ws, void* stream) {
  if (ws == nullptr) return H3ATTN_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return H3ATTN_ECUDA;
  int status = 0;
  if (cudaMemcpy(&status, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return H3ATTN_ECUDA;
  if (status != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return H3ATTN_ECUDA;
  if (status == h3::kStatusTimeout) return H3ATTN_ETIMEOUT;
  if (status == h3::kStatusData) return H3ATTN_EDATA;
  return status == 0 ? H3ATTN_OK : H3ATTN_ECUDA;
}

int h3attn_set_wait_polls(uint32_t polls) {
  g_wait_polls.store(polls, std::memory_order_relaxed);
  return H3ATTN_OK;
}

int h3attn_selftest_timeout(void* ws, uint32_t polls, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return H3ATTN_EINVAL;
  if (h3::launch_selftest_timeout(static_cast<int*>(ws), polls, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ECUDA;
  return H3ATTN_OK;
}

const char* h3attn_strerror(int status) {
  switch (status) {
    case H3ATTN_OK: return "ok";
    case H3ATTN_EINVAL: return "invalid argument";
    case H3ATTN_EUNSUPPORTED: return "unsupported shape or layout";
    case H3ATTN_EALIGN: return "pointer not aligned (16 bytes for tensors and workspace, 4 for int32/float32 arrays)";
    case H3ATTN_ECUDA: return "CUDA call or kernel launch failed";
    case H3ATTN_ETIMEOUT: return "a bounded device-side wait gave up";
    case H3ATTN_EWORKSPACE: return "workspace missing or too small";
    case H3ATTN_EDATA: return "routed list holds a block index outside the video key blocks";
    default: return "unknown status";
  }
}

}  // extern "C"
