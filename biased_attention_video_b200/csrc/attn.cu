// Fused routed attention with the bounded temporal penalty (sm_100a).
//
// Computes, per head and query row, softmax(q.k/sqrt(d) - penalty) V over the
// key blocks the row attends ("Flash Partitions for H3 native temporal
// alignment", section 1, for the score rule; "H3 SLA Attention", "How it
// works", for attending only the routed key blocks).
//
// One CTA owns a 128-row query tile = two 64-row query blocks (A: rows 0..63,
// B: rows 64..127) of one head.  It walks the union of the two blocks' key
// lists in 128-key tiles (two 64-row key blocks per tile); each query row
// masks the key blocks its own query block does not attend.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q tile once, then K and V tiles into a 2-stage ring
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 4..7  softmax: thread = one query row = one TMEM lane
// TMEM (512 columns): S0 [0,128), S1 [128,256) double-buffered scores, the
// bf16 probabilities P(j) written over the first 64 columns of S(j & 1),
// O [256, 256 + d).
// MMA issue order S(0), S(1), PV(0), S(2), PV(1), ...: tcgen05.mma ops of one
// thread run in issue order, so S(j) never overwrites P(j-2) before PV(j-2)
// has read it, and the commit after S(j) also covers PV(j-2).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace {

constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kTileRows = 128;  // query rows per CTA
constexpr int kTileKeys = 128;  // keys per KV tile
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void report(int* status, int code) { atomicCAS(status, 0, code); }

template <int D>
struct Layout {
  static constexpr int kHalves = D / 64;                 // 128-byte swizzle atoms along d
  static constexpr int kHalfBytes = kTileRows * 128;     // one d-half of a 128-row tile
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBars = kV + kStages * kTileBytes;
  // barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done, o_final, drain
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 3;
  static constexpr int kMisc = kBars + kNumBars * 8;      // tmem base, abort, n_entries
  static constexpr int kBitmaps = kMisc + 16;
  static int host_bytes(int n_blocks) {
    int nwords = (n_blocks + 31) / 32;
    return 1024 /*alignment slack*/ + kBitmaps + 2 * nwords * 4 + n_blocks * 4;
  }
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* o_final;
  uint64_t* drain;
};

__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = b + 1 + kStages;
  r.v_full = b + 1 + 2 * kStages;
  r.v_empty = b + 1 + 3 * kStages;
  r.s_full = b + 1 + 4 * kStages;
  r.p_full = b + 3 + 4 * kStages;
  r.o_done = b + 5 + 4 * kStages;
  r.o_final = b + 6 + 4 * kStages;
  r.drain = b + 7 + 4 * kStages;
  return r;
}

// Bounded wait with CTA-wide abort.  On give-up: raise the CTA abort flag and
// the global status word.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const AttnParams& p,
                                         volatile int* abort) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      if (i >= p.wait_polls || now - t0 > p.wait_ns) {
        *abort = 1;
        report(p.status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Wait used only while draining in-flight async work before exit: ignores
// the abort flag, still bounded.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const AttnParams& p) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      if (now - t0 > p.wait_ns) {
        report(p.status, kStatusTimeout);
        return;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars bars = carve_bars(smem + L::kBars);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int* n_entries_slot = reinterpret_cast<int*>(smem + L::kMisc + 8);
  const int nwords = (p.n_blocks + 31) >> 5;
  uint32_t* bm_a = reinterpret_cast<uint32_t*>(smem + L::kBitmaps);
  uint32_t* bm_b = bm_a + nwords;
  uint32_t* list = bm_b + nwords;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // Tile order: heaviest (dense) query tiles first, head-minor inside a class.
  int head, qtile;
  {
    const int lin = blockIdx.x;
    const int heavy = p.n_dense_tiles * p.H;
    if (lin < heavy) {
      head = lin % p.H;
      qtile = lin / p.H;
    } else {
      const int r = lin - heavy;
      head = r % p.H;
      qtile = p.n_dense_tiles + r / p.H;
    }
  }
  if (*reinterpret_cast<volatile int*>(p.status) == kStatusTimeout) return;  // an earlier CTA gave up

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bars.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars.k_full + s, 1);
      mbar_init(bars.k_empty + s, 1);
      mbar_init(bars.v_full + s, 1);
      mbar_init(bars.v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars.s_full + b, 1);
      mbar_init(bars.p_full + b, 128);
    }
    mbar_init(bars.o_done, 1);
    mbar_init(bars.o_final, 1);
    mbar_init(bars.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, 512);
    tmem_relinquish();
  }

  // ---- key-block list of this tile: union of the two query blocks' lists ----
  const int qb_a = 2 * qtile, qb_b = 2 * qtile + 1;
  const bool has_a = qb_a < p.n_blocks, has_b = qb_b < p.n_blocks;
  const bool dense_a = p.kv_sel == nullptr || qb_a < p.first_video_block;
  const bool dense_b = p.kv_sel == nullptr || qb_b < p.first_video_block;
  for (int w = tid; w < nwords; w += kThreads) {
    const int lo = w * 32;
    uint32_t full = (p.n_blocks - lo >= 32) ? 0xFFFFFFFFu : ((1u << (p.n_blocks - lo)) - 1u);
    int nf = p.first_video_block - lo;
    uint32_t forced = nf <= 0 ? 0u : (nf >= 32 ? 0xFFFFFFFFu : ((1u << nf) - 1u));
    bm_a[w] = !has_a ? 0u : (dense_a ? full : forced);
    bm_b[w] = !has_b ? 0u : (dense_b ? full : forced);
  }
  __syncthreads();
  if (has_a && !dense_a) {
    const int32_t* lst = p.kv_sel + ((size_t)head * p.n_video_blocks + (qb_a - p.first_video_block)) * p.k;
    for (int i = tid; i < p.k; i += kThreads) {
      int e = lst[i];
      if (e < p.first_video_block || e >= p.n_blocks) report(p.status, kStatusData);
      else atomicOr(bm_a + (e >> 5), 1u << (e & 31));
    }
  }
  if (has_b && !dense_b) {
    const int32_t* lst = p.kv_sel + ((size_t)head * p.n_video_blocks + (qb_b - p.first_video_block)) * p.k;
    for (int i = tid; i < p.k; i += kThreads) {
      int e = lst[i];
      if (e < p.first_video_block || e >= p.n_blocks) report(p.status, kStatusData);
      else atomicOr(bm_b + (e >> 5), 1u << (e & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    // lane l owns words [l*per, (l+1)*per)
    const int per = (nwords + 31) / 32;
    int cnt = 0;
    for (int w = lane * per; w < min(nwords, (lane + 1) * per); ++w) cnt += __popc(bm_a[w] | bm_b[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = incl - cnt;
    for (int w = lane * per; w < min(nwords, (lane + 1) * per); ++w) {
      uint32_t a = bm_a[w], b = bm_b[w], u = a | b;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        list[pos++] = (uint32_t)(w * 32 + bit) | (((a >> bit) & 1u) << 16) | (((b >> bit) & 1u) << 17);
      }
    }
    if (lane == 31) *n_entries_slot = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  const int n_entries = *n_entries_slot;
  const int n_tiles = (n_entries + 1) >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued_k[kStages] = {0, 0}, issued_v[kStages] = {0, 0};
      const int q_row0 = qtile * kTileRows;
      uint8_t* sq = smem + L::kQ;
      mbar_arrive_expect_tx(bars.q_full, L::kTileBytes);
#pragma unroll
      for (int c = 0; c < L::kHalves; ++c) {
        tma_load_3d(sq + c * L::kHalfBytes, &tm_q, bars.q_full, c * 64, q_row0, head);
        tma_load_3d(sq + c * L::kHalfBytes + 8192, &tm_q, bars.q_full, c * 64, q_row0 + 64, head);
      }
      const int oob_row = p.n_blocks * 64;  // a whole block past S: zero-filled by TMA
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        const int e0 = (int)(list[2 * j] & 0xFFFFu);
        const int e1 = (2 * j + 1 < n_entries) ? (int)(list[2 * j + 1] & 0xFFFFu) : -1;
        const int r0 = e0 * 64, r1 = e1 >= 0 ? e1 * 64 : oob_row;
        if (!wait_bar(bars.k_empty + s, ph ^ 1u, p, abort_flag)) break;
        uint8_t* sk = smem + L::kK + s * L::kTileBytes;
        mbar_arrive_expect_tx(bars.k_full + s, L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kHalves; ++c) {
          tma_load_3d(sk + c * L::kHalfBytes, &tm_k, bars.k_full + s, c * 64, r0, head);
          tma_load_3d(sk + c * L::kHalfBytes + 8192, &tm_k, bars.k_full + s, c * 64, r1, head);
        }
        ++issued_k[s];
        if (!wait_bar(bars.v_empty + s, ph ^ 1u, p, abort_flag)) break;
        uint8_t* sv = smem + L::kV + s * L::kTileBytes;
        mbar_arrive_expect_tx(bars.v_full + s, L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kHalves; ++c) {
          tma_load_3d(sv + c * L::kHalfBytes, &tm_v, bars.v_full + s, c * 64, r0, head);
          tma_load_3d(sv + c * L::kHalfBytes + 8192, &tm_v, bars.v_full + s, c * 64, r1, head);
        }
        ++issued_v[s];
      }
      // drain: every issued load must land before the CTA may exit
      drain_wait(bars.q_full, 0, p);
      for (int s = 0; s < kStages; ++s) {
        if (issued_k[s]) drain_wait(bars.k_full + s, (issued_k[s] - 1) & 1u, p);
        if (issued_v[s]) drain_wait(bars.v_full + s, (issued_v[s] - 1) & 1u, p);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, kTileKeys, 0, 0);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t tmem_o = tmem_base + 256;
      bool ok = wait_bar(bars.q_full, 0, p, abort_flag);
      auto issue_pv = [&](int jj) -> bool {
        const int s = jj % kStages;
        const uint32_t ph = (uint32_t)(jj / kStages) & 1u;
        if (!wait_bar(bars.p_full + (jj & 1), (uint32_t)(jj >> 1) & 1u, p, abort_flag)) return false;
        if (!wait_bar(bars.v_full + s, ph, p, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + L::kV + s * L::kTileBytes);
        const uint32_t p_tmem = tmem_base + (uint32_t)(jj & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk) {
          // B = V tile, MN-major: 16 keys per step = two 8-row swizzle groups
          const uint64_t bdesc = sw128_desc(v_addr + kk * 2048, L::kHalfBytes, 1024);
          umma_ts(tmem_o, p_tmem + kk * 8, bdesc, kIdescO, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bars.o_done);
        umma_commit(bars.v_empty + s);
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        if (!wait_bar(bars.k_full + s, ph, p, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + L::kK + s * L::kTileBytes);
        const uint32_t s_tmem = tmem_base + (uint32_t)(j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t adesc = sw128_desc(q_addr + c * L::kHalfBytes + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(k_addr + c * L::kHalfBytes + off, 16, 1024);
          umma_ss(s_tmem, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bars.s_full + (j & 1));
        umma_commit(bars.k_empty + s);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n_tiles > 0) ok = issue_pv(n_tiles - 1);
      umma_commit(bars.o_final);
      // drain: all issued MMAs complete before TMEM is released
      umma_commit(bars.drain);
      drain_wait(bars.drain, 0, p);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int r = tid - 128;  // row within the tile == TMEM lane
    const int quarter = warp & 3;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const int my_half = r >> 6;  // 0: query block A, 1: query block B
    const int qrow = qtile * kTileRows + r;
    const bool row_valid = qrow < p.S;
    const bool pen_row = p.pen_on && row_valid && p.seg[qrow] == kSegOutput;
    const float tq = pen_row ? p.times[qrow] : 0.0f;
    const float scale = p.scale_log2;
    float m = -INFINITY;  // running max, log2 units (upper bound of the true max)
    float l = 0.0f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective (.sync.aligned): every branch that
    // guards one is made warp-uniform with __all_sync / __any_sync.
    constexpr unsigned kFull = 0xFFFFFFFFu;
    for (int j = 0; j < n_tiles; ++j) {
      const int buf = j & 1;
      const bool got = wait_bar(bars.s_full + buf, (uint32_t)(j >> 1) & 1u, p, abort_flag);
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTileKeys];
      {
        uint32_t tmp[32];
#pragma unroll
        for (int c = 0; c < kTileKeys / 32; ++c) {
          __syncwarp();
          tmem_ld32(tmem_base + lane_addr + (uint32_t)buf * 128 + c * 32, tmp);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(tmp[i]);
        }
      }
      // per 64-key half: attended? penalty mode? valid keys?
      int mode[2];      // 0 skip, 1 plain, 2 constant penalty, 3 per-key penalty
      int nvalid[2];
      float cpen[2];
      int kblock[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int idx = 2 * j + hh;
        mode[hh] = 0;
        nvalid[hh] = 0;
        cpen[hh] = 0.0f;
        kblock[hh] = 0;
        if (idx < n_entries) {
          const uint32_t ent = list[idx];
          const bool att = ((ent >> (16 + my_half)) & 1u) != 0;
          const int b = (int)(ent & 0xFFFFu);
          kblock[hh] = b;
          if (att) {
            const uint2 kd = p.kv_desc[b];
            nvalid[hh] = (int)(kd.x & 0xFFu);
            const int kind = (int)((kd.x >> 8) & 3u);
            mode[hh] = 1;
            if (pen_row && kind == 1) {
              const float dt = fabsf(tq - __uint_as_float(kd.y));
              const float ex = fmaxf(dt - p.window, 0.0f) * p.inv_falloff;
              cpen[hh] = fminf(p.strength_log2 * ex * ex, p.cap_log2);
              mode[hh] = 2;
            } else if (pen_row && kind == 2) {
              mode[hh] = 3;
            }
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (mode[hh] == 0) continue;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < nvalid[hh]) mx = fmaxf(mx, sv[hh * 64 + i]);
      }
      mx *= scale;
      // Conditional rescale: the running max only moves when it grows by more
      // than 2^8; below that the stale max keeps every probability <= 256.
      const bool grow = mx > m + kRescaleThreshold;
      const bool o_rescale = grow && l > 0.0f;
      if (__any_sync(kFull, o_rescale)) {
        // O holds PV(0..j-1): wait for PV(j-1), then scale it in place
        // (lanes that do not rescale multiply by 1).
        const bool got2 = wait_bar(bars.o_done, (uint32_t)(j - 1) & 1u, p, abort_flag);
        if (!__all_sync(kFull, got2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float alpha = o_rescale ? ex2(m - mx) : 1.0f;
        uint32_t tmp[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint32_t a = tmem_base + lane_addr + 256 + c * 32;
          __syncwarp();
          tmem_ld32(a, tmp);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) tmp[i] = __float_as_uint(__uint_as_float(tmp[i]) * alpha);
          tmem_st32(a, tmp);
        }
        tmem_wait_st();
        l *= alpha;
      }
      if (grow) m = mx;
      // probabilities -> bf16 pairs into the first 64 columns of S(buf)
#pragma unroll
      for (int c = 0; c < kTileKeys / 32; ++c) {
        const int hh = c >> 1;
        uint32_t packed[16];
        float pr[32];
        const int md = mode[hh];
        if (md == 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pr[i] = 0.0f;
        } else if (md == 3) {
          const int key0 = kblock[hh] * 64 + (c & 1) * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = (c & 1) * 32 + i;
            float pen_k = 0.0f;
            if (col < nvalid[hh] && p.seg[key0 + i] == kSegGuide) {
              const float dt = fabsf(tq - p.times[key0 + i]);
              const float ex = fmaxf(dt - p.window, 0.0f) * p.inv_falloff;
              pen_k = fminf(p.strength_log2 * ex * ex, p.cap_log2);
            }
            pr[i] = col < nvalid[hh] ? ex2(fmaf(sv[c * 32 + i], scale, -(m + pen_k))) : 0.0f;
          }
        } else {
          const float off = -(m + cpen[hh]);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = (c & 1) * 32 + i;
            pr[i] = col < nvalid[hh] ? ex2(fmaf(sv[c * 32 + i], scale, off)) : 0.0f;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          l += pr[2 * i] + pr[2 * i + 1];
          packed[i] = pack_bf16(pr[2 * i], pr[2 * i + 1]);
        }
        __syncwarp();
        tmem_st16(tmem_base + lane_addr + (uint32_t)buf * 128 + c * 16, packed);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full + buf);
    }
    // ---------------------------------------------------------- epilogue
    bool fin = __all_sync(kFull, ok) && n_tiles > 0;
    if (fin) fin = wait_bar(bars.o_final, 0, p, abort_flag);
    if (__all_sync(kFull, fin)) {
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      uint16_t* orow = p.o + ((size_t)head * p.S + (row_valid ? qrow : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t tmp[32];
        __syncwarp();
        tmem_ld32(tmem_base + lane_addr + 256 + c * 32, tmp);
        tmem_wait_ld();
        uint32_t outw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          outw[i] = pack_bf16(__uint_as_float(tmp[2 * i]) * inv_l, __uint_as_float(tmp[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
        }
      }
      if (row_valid && p.lse != nullptr) p.lse[(size_t)head * p.S + qrow] = (m + __log2f(l)) * kLn2;
    }
  }
  // warps 2..3 have no role after the list is built

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace

int attn_smem_bytes(int d, int n_blocks) {
  return d == 64 ? Layout<64>::host_bytes(n_blocks) : Layout<128>::host_bytes(n_blocks);
}

cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnParams& p, int n_ctas, cudaStream_t stream) {
  const int smem = attn_smem_bytes(p.d, p.n_blocks);
  if (p.d == 64) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel<64><<<n_ctas, kThreads, smem, stream>>>(tq, tk, tv, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel<128><<<n_ctas, kThreads, smem, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

}  // namespace h3
