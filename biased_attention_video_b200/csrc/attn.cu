// Fused routed attention with the bounded temporal penalty (sm_100a).
//
// Computes, per head and query row, softmax(q.k/sqrt(d) - penalty) V over the
// key blocks the row attends ("Flash Partitions for H3 native temporal
// alignment", section 1, for the score rule; "H3 SLA Attention", "How it
// works", for attending only the routed key blocks).
//
// One CTA owns a 128-row query tile = two 64-row query blocks (A: rows 0..63,
// B: rows 64..127) of one head: adjacent blocks over the dense prefix, a pair
// chosen by routed-list overlap elsewhere.  It walks the union of the two
// blocks' key lists in 128-key tiles (two 64-row key blocks per tile); each
// query row masks the key blocks its own query block does not attend, and a
// softmax warp whose query block skips a key block writes zero probabilities
// for it without reading its scores.
//
// Two CTAs share an SM (TMEM 256 columns and < 114 KB of shared memory each),
// so one CTA's tensor-core work overlaps the other's softmax.
//
// A second instantiation (kQK8) takes Q and K as int8 codes with per-token
// scales: the S products run as int8 MMAs, everything else is shared.
//
// Warp roles (320 threads; two CTAs per SM leave 96 registers per thread):
//   warp 0      TMA producer: Q tile once, then K and V 128-key tiles
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 2..9  softmax: two threads per query row (= TMEM lane); the thread
//               of part p owns key block p of every tile (keys 64p..64p+63);
//               warp w may only touch TMEM lanes [32 (w % 4), 32 (w % 4) + 32)
//
// TMEM: S [0,128) fp32 scores of the current tile; O [128, 128 + d).
// Each softmax thread reads all 64 scores of its key block, takes their max
// and exchanges it once with its partner thread; then it works in two phases:
//   phase 0, keys 0..47 of its block: bf16 probabilities go back into TMEM
//            over the block's first 24 score columns (TS-form PV);
//   phase 1, keys 48..63: probabilities go to an 8 KB shared-memory tile
//            (SS-form PV).
// Before handing phase 0 over, each thread has read its phase-1 scores again,
// so the whole S region is free once PV(j, phase 0) has read its P:
// the MMA warp issues S(j+1) right behind PV(j, phase 0), and the next tile's
// scores are computed while the softmax still works on phase 1 of this one.
// MMA issue order: S(0) | PV(0,0) S(1) PV(0,1) | PV(1,0) S(2) PV(1,1) | ...
// The tcgen05.mma ops of one thread run in issue order, so S(j+1) never
// overwrites P(j, phase 0) before PV(j, phase 0) has read it, and when the
// commit after S(j+1) fires, PV(j, phase 0) is complete too.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "fastmath.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "softmax.cuh"

namespace h3 {
namespace {

using namespace sm;

constexpr int kThreads = 320;
constexpr int kTileRows = 128;  // query rows per CTA
constexpr int kTileKeys = 128;  // keys per KV tile
constexpr int kPhase0Keys = 48;  // keys per block whose P stays in TMEM
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 128;  // O column offset

template <int D, bool kQK8>
struct Layout {
  static constexpr int kHalves = D / 64;               // 128-byte swizzle atoms along d (bf16 V)
  static constexpr int kHalfBytes = kTileRows * 128;   // one 128-byte-wide column of a 128-row tile
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  // Q and K: bf16, or int8 codes (one 128-byte atom holds d = 128)
  static constexpr int kQKHalves = kQK8 ? D / 128 : D / 64;
  static constexpr int kQKElems = kQK8 ? 128 : 64;  // elements per 128-byte atom
  static constexpr int kQKTileBytes = kQKHalves * kHalfBytes;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQKTileBytes;
  static constexpr int kV = kK + kQKTileBytes;
  // phase-1 probabilities: two K-major 32-byte-swizzled operands (one per key
  // block of the tile), 128 rows x 16 keys each
  static constexpr int kPh1 = kV + kTileBytes;
  static constexpr int kPh1StepBytes = kTileRows * 32;
  static constexpr int kBars = kPh1 + 2 * kPh1StepBytes;
  // q_full, k_full, k_empty, v_full, v_empty, s_full, p_full[2], o_done, o_final, drain, xchg[4]
  static constexpr int kNumBars = 15;
  static constexpr int kMisc = kBars + kNumBars * 8;  // tmem base, abort flag, n_entries, n_fast
  static constexpr int kRed = kMisc + 16;             // partial row maxima / sums: float [2][2][128]
  static constexpr int kBitmaps = kRed + 2 * 2 * 128 * 4;
  static int host_bytes(int n_blocks) {
    const int nwords = (n_blocks + 31) / 32;
    return 1024 /*alignment slack*/ + kBitmaps + 2 * nwords * 4 + ((n_blocks * 2 + 15) & ~15);
  }
};

struct Bars {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done, *o_final, *drain, *xchg;
};

// p_full[ph]: P of phase ph of the current tile is in place (one completion
// per tile each, so a waiter is never more than one phase behind).
// o_done: PV(j, phase 1) complete, hence all of tile j's MMAs (one thread
// issues them, and they run in issue order).  The softmax waits for it on
// every tile (o_done(j-1) in phase 0 of tile j), so its parity never falls
// behind.
// xchg[q]: the two softmax warps of TMEM lane quarter q have written their
// partial row values (64 arrivals per exchange; neither warp can run more than
// one exchange ahead of the other).
__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  return Bars{b, b + 1, b + 2, b + 3, b + 4, b + 5, b + 6, b + 8, b + 9, b + 10, b + 11};
}

// kQK8: Q and K arrive as int8 codes with per-token scales (p.q_scale,
// p.k_scale); S = Q K^T runs as int8 MMAs into s32 and is scaled back per
// query row and key in the softmax.
template <int D, bool kQK8>
__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  static_assert(!kQK8 || D == 128, "int8 QK needs d = 128 (one 128-byte atom per row)");
  using L = Layout<D, kQK8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars bars = carve_bars(smem + L::kBars);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int* n_entries_slot = reinterpret_cast<int*>(smem + L::kMisc + 8);
  int* n_fast_slot = reinterpret_cast<int*>(smem + L::kMisc + 12);
  const int nwords = (p.n_blocks + 31) >> 5;
  uint32_t* bm_a = reinterpret_cast<uint32_t*>(smem + L::kBitmaps);
  uint32_t* bm_b = bm_a + nwords;
  // entry = key block (14 bits) | attended by block A << 14 | attended by block B << 15
  uint16_t* list = reinterpret_cast<uint16_t*>(bm_b + nwords);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // Tile order: head-major, so the ~300 CTAs resident at a time share one or
  // two heads' K/V in L2; inside a head the dense (prefix) query tiles come
  // first, so the longest tiles start earliest.
  const int n_qtiles = p.n_dense_tiles + p.n_paired_tiles;
  const int head = (int)(blockIdx.x / n_qtiles);
  const int qtile = (int)(blockIdx.x % n_qtiles);
  // An earlier CTA that gave up leaves the status word set: skip the work
  // (decided once per CTA so that every thread leaves together).
  if (tid == 0) *abort_flag = *reinterpret_cast<volatile int*>(p.status) == kStatusTimeout ? 1 : 0;
  __syncthreads();
  if (*abort_flag) return;
  __syncthreads();

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bars.q_full, 1);
    mbar_init(bars.k_full, 1);
    mbar_init(bars.k_empty, 1);
    mbar_init(bars.v_full, 1);
    mbar_init(bars.v_empty, 1);
    mbar_init(bars.s_full, 1);
    mbar_init(bars.p_full, 8);
    mbar_init(bars.p_full + 1, 8);
    mbar_init(bars.o_done, 1);
    mbar_init(bars.o_final, 1);
    mbar_init(bars.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(bars.xchg + q, 64);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }

  // ---- the tile's two query blocks: adjacent ones over the dense prefix,
  // else the pair chosen by routed-list overlap (qb_b = -1: block a alone)
  int qb_a = 2 * qtile, qb_b = 2 * qtile + 1;
  if (qtile >= p.n_dense_tiles) {
    const uint32_t e = __ldg(p.qpairs + (size_t)head * p.n_paired_tiles + (qtile - p.n_dense_tiles));
    qb_a = (int)(e & 0xFFFFu);
    qb_b = (e >> 16) == kNoPair ? -1 : (int)(e >> 16);
  }
  const bool has_a = qb_a < p.n_blocks, has_b = qb_b >= 0 && qb_b < p.n_blocks;

  // ---- key-block list of this tile: union of the two query blocks' lists ----
  const bool dense_a = p.kv_sel == nullptr || qb_a < p.first_video_block;
  const bool dense_b = p.kv_sel == nullptr || qb_b < p.first_video_block;
  for (int w = tid; w < nwords; w += kThreads) {
    const int lo = w * 32;
    const uint32_t full = (p.n_blocks - lo >= 32) ? 0xFFFFFFFFu : ((1u << (p.n_blocks - lo)) - 1u);
    const int nf = p.first_video_block - lo;
    const uint32_t forced = nf <= 0 ? 0u : (nf >= 32 ? 0xFFFFFFFFu : ((1u << nf) - 1u));
    bm_a[w] = !has_a ? 0u : (dense_a ? full : forced);
    bm_b[w] = !has_b ? 0u : (dense_b ? full : forced);
  }
  __syncthreads();
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int qb = half == 0 ? qb_a : qb_b;
    const bool routed = half == 0 ? (has_a && !dense_a) : (has_b && !dense_b);
    uint32_t* bm = half == 0 ? bm_a : bm_b;
    if (routed) {
      const int32_t* lst = p.kv_sel + ((size_t)head * p.n_video_blocks + (qb - p.first_video_block)) * p.k;
      for (int i = tid; i < p.k; i += kThreads) {
        const int e = lst[i];
        if (e < p.first_video_block || e >= p.n_blocks) report(p.status, kStatusData);
        else atomicOr(bm + (e >> 5), 1u << (e & 31));
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // Entries in ascending block order, except that the blocks needing
    // per-key treatment (p.slow_blocks) go after all the others; the online
    // softmax may visit key blocks in any order.  Lane l owns words
    // [l*per, (l+1)*per); fast and slow counts share one scan (16 bits each).
    const int per = (nwords + 31) / 32;
    const int w0 = lane * per, w1 = min(nwords, (lane + 1) * per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) {
      const uint32_t u = bm_a[w] | bm_b[w], slow = p.slow_blocks[w];
      cnt += __popc(u & ~slow) | (__popc(u & slow) << 16);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    const int n_fast = __shfl_sync(kFull, incl, 31) & 0xFFFF;
    int pos_f = (incl - cnt) & 0xFFFF, pos_s = n_fast + ((incl - cnt) >> 16);
    for (int w = w0; w < w1; ++w) {
      const uint32_t a = bm_a[w], b = bm_b[w], slow = p.slow_blocks[w];
      uint32_t u = a | b;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        const uint16_t e = (uint16_t)((w * 32 + bit) | (((a >> bit) & 1u) << 14) | (((b >> bit) & 1u) << 15));
        if ((slow >> bit) & 1u) list[pos_s++] = e;
        else list[pos_f++] = e;
      }
    }
    if (lane == 31) {
      *n_entries_slot = (incl & 0xFFFF) + (incl >> 16);
      *n_fast_slot = incl & 0xFFFF;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  const int n_entries = *n_entries_slot;
  const int n_tiles = (n_entries + 1) >> 1;
  const int n_fast_tiles = *n_fast_slot >> 1;  // tiles whose two blocks are both fast

  if (warp < 2) {
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t issued_k = 0, issued_v = 0;
      const int oob_row = p.n_blocks * 64;  // a whole block past S: zero-filled by TMA
      const int qa_row = has_a ? qb_a * 64 : oob_row, qb_row = has_b ? qb_b * 64 : oob_row;
      uint8_t* sq = smem + L::kQ;
      uint8_t* sk = smem + L::kK;
      uint8_t* sv = smem + L::kV;
      mbar_arrive_expect_tx(bars.q_full, L::kQKTileBytes);
#pragma unroll
      for (int c = 0; c < L::kQKHalves; ++c) {
        tma_load_3d(sq + c * L::kHalfBytes, &tm_q, bars.q_full, c * L::kQKElems, qa_row, head);
        tma_load_3d(sq + c * L::kHalfBytes + 8192, &tm_q, bars.q_full, c * L::kQKElems, qb_row, head);
      }
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t ph = (uint32_t)j & 1u;
        const int r0 = (int)(list[2 * j] & 0x3FFFu) * 64;
        const int r1 = (2 * j + 1 < n_entries) ? (int)(list[2 * j + 1] & 0x3FFFu) * 64 : oob_row;
        if (!wait_bar(bars.k_empty, ph ^ 1u, p, abort_flag)) break;
        mbar_arrive_expect_tx(bars.k_full, L::kQKTileBytes);
#pragma unroll
        for (int c = 0; c < L::kQKHalves; ++c) {
          tma_load_3d(sk + c * L::kHalfBytes, &tm_k, bars.k_full, c * L::kQKElems, r0, head);
          tma_load_3d(sk + c * L::kHalfBytes + 8192, &tm_k, bars.k_full, c * L::kQKElems, r1, head);
        }
        ++issued_k;
        if (!wait_bar(bars.v_empty, ph ^ 1u, p, abort_flag)) break;
        mbar_arrive_expect_tx(bars.v_full, L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kHalves; ++c) {
          tma_load_3d(sv + c * L::kHalfBytes, &tm_v, bars.v_full, c * 64, r0, head);
          tma_load_3d(sv + c * L::kHalfBytes + 8192, &tm_v, bars.v_full, c * 64, r1, head);
        }
        ++issued_v;
      }
      // drain: every issued load must land before the CTA may exit
      drain_wait(bars.q_full, 0, p);
      if (issued_k) drain_wait(bars.k_full, (issued_k - 1) & 1u, p);
      if (issued_v) drain_wait(bars.v_full, (issued_v - 1) & 1u, p);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescS = kQK8 ? idesc_s8_s32(128, kTileKeys) : idesc_bf16_f32(128, kTileKeys, 0, 0);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      const uint32_t ph1_addr = smem_u32(smem + L::kPh1);
      const uint32_t tmem_s = tmem_base;
      const uint32_t tmem_o = tmem_base + kTmemO;
      auto issue_s = [&](int j) -> bool {
        if (!wait_bar(bars.k_full, (uint32_t)j & 1u, p, abort_flag)) return false;
        tc_fence_after();
        // one MMA per 32-byte K step: 16 bf16 or 32 int8 elements of d
#pragma unroll
        for (int kk = 0; kk < L::kQKHalves * 4; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t adesc = sw128_desc(q_addr + c * L::kHalfBytes + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(k_addr + c * L::kHalfBytes + off, 16, 1024);
          if constexpr (kQK8)
            umma_ss_i8(tmem_s, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
          else
            umma_ss(tmem_s, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bars.s_full);
        umma_commit(bars.k_empty);
        return true;
      };
      bool ok = wait_bar(bars.q_full, 0, p, abort_flag);
      if (ok && n_tiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const uint32_t ph = (uint32_t)j & 1u;
        if (!wait_bar(bars.v_full, ph, p, abort_flag) || !wait_bar(bars.p_full, ph, p, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // PV(j, phase 0): keys 16c..16c+15 of block b (c < 3) = V rows 64b+16c..,
        // P in TMEM columns 64b + 8c (B = V tile, MN-major: 16 keys per step)
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
          for (int c = 0; c < kPhase0Keys / 16; ++c) {
            const uint64_t bdesc = sw128_desc(v_addr + (4 * b + c) * 2048, L::kHalfBytes, 1024);
            umma_ts(tmem_o, tmem_s + 64 * b + 8 * c, bdesc, kIdescO, (j > 0 || b > 0 || c > 0) ? 1u : 0u);
          }
        // S(j+1): every thread has read its phase-1 scores before p_full[0]
        if (j + 1 < n_tiles && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        if (!wait_bar(bars.p_full + 1, ph, p, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // PV(j, phase 1): keys 48..63 of block b, P from shared memory
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint64_t adesc = sw32_kmajor_desc(ph1_addr + b * L::kPh1StepBytes);
          const uint64_t bdesc = sw128_desc(v_addr + (4 * b + 3) * 2048, L::kHalfBytes, 1024);
          umma_ss(tmem_o, adesc, bdesc, kIdescO, 1u);
        }
        umma_commit(bars.v_empty);
        umma_commit(bars.o_done);
      }
      umma_commit(bars.o_final);
      // drain: all issued MMAs complete before TMEM is released
      umma_commit(bars.drain);
      drain_wait(bars.drain, 0, p);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Two threads per query row: warp w handles TMEM lanes [32 (w % 4), +32)
    // and key block part = (w - 2) / 4 of every tile.  The two threads of a
    // row exchange their partial maxima once per tile through shared memory
    // (an mbarrier per lane quarter), so both apply the same running max; each
    // rescales and finally normalises its half of O's columns.
    // tcgen05.ld/st are warp-collective (.sync.aligned): every branch that
    // guards one is made warp-uniform with __all_sync / __any_sync.
    constexpr int kOCols = D / 2;  // O columns per thread
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem_base + lane_addr + (uint32_t)(64 * part);  // this thread's block of S
    const uint32_t t_o = tmem_base + lane_addr + kTmemO + (uint32_t)(part * kOCols);
    uint64_t* xbar = bars.xchg + quarter;
    uint32_t n_xchg = 0;  // exchanges done (phase parity of xbar)
    float* red = reinterpret_cast<float*>(smem + L::kRed);  // [2 slots][2 parts][128 rows]
    // phase-1 probabilities of this row: 32 bytes at row r of this part's operand
    uint8_t* ph1_row = smem + L::kPh1 + part * L::kPh1StepBytes + r * 32;
    const uint32_t ph1_swz = (uint32_t)((r >> 2) & 1) << 4;  // 32-byte swizzle: bit 4 ^= bit 7
    const int my_bit = 14 + (r >> 6);  // list bit of this row's query block
    const int qrow = (r < 64 ? qb_a : qb_b) * 64 + (r & 63);
    const bool row_valid = (r < 64 ? has_a : has_b) && qrow < p.S;
    const bool pen_row = p.pen_on && row_valid && p.seg[qrow] == kSegOutput;
    const float tq = pen_row ? p.times[qrow] : 0.0f;
    // log2-units multiplier of this row's scores; with int8 QK it also
    // carries the row's quantisation scale (the key's is applied per score)
    const float scale = kQK8 ? (row_valid ? p.q_scale[(size_t)head * p.scale_stride + qrow] : 0.0f) * p.scale_log2
                             : p.scale_log2;
    float m = -INFINITY;  // running max, log2 units (upper bound of the true max)
    float l = 0.0f;       // partial row sum over this thread's keys
    bool ok = true;

    // Combine this thread's partial max with its partner's.  Exchanges
    // alternate between two slots: a thread writes slot s again only after
    // passing the next exchange's barrier, which its partner reaches only
    // after reading slot s.  Returns false on give-up.
    auto exchange_max = [&](float pmax, int slot, float& mx) -> bool {
      red[(slot * 2 + part) * 128 + r] = pmax;
      mbar_arrive(xbar);
      const bool gotx = wait_bar(xbar, n_xchg & 1u, p, abort_flag);
      ++n_xchg;
      if (!__all_sync(kFull, gotx)) return false;
      mx = fmaxf(pmax, red[(slot * 2 + (part ^ 1)) * 128 + r]) * scale;
      return true;
    };
    // O *= alpha for this thread's O columns (warp-uniform call)
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int c = 0; c < kOCols / 16; ++c) {
        uint32_t tmp[16];
        __syncwarp();
        tmem_ld16(t_o + c * 16, tmp);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) tmp[i] = __float_as_uint(__uint_as_float(tmp[i]) * alpha);
        tmem_st16(t_o + c * 16, tmp);
      }
    };

    // The tile for a warp whose rows do not attend this thread's key block.
    auto skip_tile = [&](int j) -> bool {
      const uint32_t ph = (uint32_t)j & 1u;
      const uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int g = 0; g < kPhase0Keys / 16; ++g) {
        __syncwarp();
        tmem_st8(t_s + 8 * g, zero);
      }
      float mx;
      if (!exchange_max(-INFINITY, j & 1, mx)) return false;
      const bool grow = mx > m + kRescaleThreshold;
      const bool o_rescale = grow && m > -INFINITY;
      const float m_old = m;
      if (grow) m = mx;
      if (j > 0) {
        if (!__all_sync(kFull, wait_bar(bars.o_done, ph ^ 1u, p, abort_flag))) return false;
        tc_fence_after();
      }
      float alpha = 1.0f;
      if (__any_sync(kFull, o_rescale)) {
        alpha = o_rescale ? ex2(m_old - m) : 1.0f;
        rescale_o(alpha);
      }
      l *= alpha;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full);
      *reinterpret_cast<uint4*>(ph1_row) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(ph1_row + 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full + 1);
      return true;
    };

    // One tile; kGeneral selects the per-key path (validity, per-key penalty)
    // that the few slow key blocks need -- kept out of the loop over the
    // others so that it does not weigh on their register allocation.
    auto tile = [&](int j, auto general) -> bool {
      constexpr bool kGeneral = decltype(general)::value;
      const uint32_t ph = (uint32_t)j & 1u;
      // this thread's key block and its descriptor, fetched before the wait
      const int idx = 2 * j + part;
      const uint32_t ent = idx < n_entries ? (uint32_t)list[idx] : 0u;
      const bool attended = idx < n_entries && ((ent >> my_bit) & 1u);
      const uint4 kd = attended ? __ldg(p.kv_desc + (ent & 0x3FFFu)) : make_uint4(0u, 0u, 0u, 0u);
      BlockMode bm{0, 0, (int)(ent & 0x3FFFu) * 64, 64, 0.0f, 0.0f};
      if (attended) {
        bm.nv = (int)(kd.x & 0xFFu);
        const int kind = (int)((kd.x >> 8) & 3u);
        bm.mode = 1;
        if (pen_row && kind == 1) {
          // a non-guide run has time NaN: its penalty evaluates to 0
          bm.split = (int)((kd.x >> 16) & 0xFFu);
          bm.pen_a = block_penalty_log2(tq, __uint_as_float(kd.y), p);
          bm.pen_b = bm.split < bm.nv ? block_penalty_log2(tq, __uint_as_float(kd.z), p) : bm.pen_a;
          bm.mode = 2;
        } else if (pen_row && kind == 2) {
          bm.mode = 3;
        }
      }
      if (!__all_sync(kFull, wait_bar(bars.s_full, ph, p, abort_flag))) {
        return false;
      }
      tc_fence_after();
      // A warp's 32 rows belong to one query block: when that block does not
      // attend this key block (the tile's other block does), the warp writes
      // zero probabilities without reading the scores; it still takes part in
      // the exchange and in any rescale of its rows.
      if (__all_sync(kFull, !attended)) return skip_tile(j);

      // All 64 scores of this thread's block: one max and one partner
      // exchange per tile, for both phases (the phase-1 scores are read
      // again after phase 0, to keep them out of phase 0's registers).
      float sv[kPhase0Keys], sv1[16];
      {
        uint32_t t32[32], t16[16], u16[16];
        __syncwarp();
        tmem_ld32(t_s, t32);
        tmem_ld16(t_s + 32, t16);
        tmem_ld16(t_s + kPhase0Keys, u16);
        tmem_wait_ld();
        if constexpr (kQK8) {
          const float* ks = p.k_scale + ((size_t)head * p.scale_stride + bm.key0);
          qk8_scores<32>(t32, ks, sv);
          qk8_scores<16>(t16, ks + 32, sv + 32);
          qk8_scores<16>(u16, ks + kPhase0Keys, sv1);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[i] = __uint_as_float(t32[i]);
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[32 + i] = __uint_as_float(t16[i]);
#pragma unroll
          for (int i = 0; i < 16; ++i) sv1[i] = __uint_as_float(u16[i]);
        }
      }
      float mx;
      const float pmax = kGeneral ? fmaxf(part_max<kPhase0Keys>(sv, bm, 0), part_max<16>(sv1, bm, kPhase0Keys))
                                  : fmaxf(full_max<kPhase0Keys>(sv, bm), full_max<16>(sv1, bm));
      if (!exchange_max(pmax, j & 1, mx)) return false;
      // Conditional rescale: the running max only moves when it grows by more
      // than 2^8; below that the stale max keeps every probability <= 256.
      const bool grow = mx > m + kRescaleThreshold;
      const bool o_rescale = grow && m > -INFINITY;
      const float m_old = m;
      if (grow) m = mx;

      // ---------------- phase 0: keys 0..47 of the block, P back into TMEM
      float lt = 0.0f;
#pragma unroll
      for (int g = 0; g < kPhase0Keys / 16; ++g) {
        uint32_t pk[8];
        lt += kGeneral ? probs16_general(sv + 16 * g, bm, 16 * g, m, scale, tq, p, pk)
                       : probs16_fast(sv + 16 * g, fast_offset(bm, 16 * g, m), scale, pk);
        __syncwarp();
        tmem_st8(t_s + 8 * g, pk);  // P of keys 16g..16g+15 over score columns 8g..8g+7
      }
      // phase-1 scores again: S(j+1) may overwrite the S region as soon as
      // PV(j, phase 0) has consumed P, which follows p_full[0]
      {
        uint32_t t16[16];
        __syncwarp();
        tmem_ld16(t_s + kPhase0Keys, t16);
        tmem_wait_ld();
        if constexpr (kQK8) {
          qk8_scores<16>(t16, p.k_scale + ((size_t)head * p.scale_stride + bm.key0 + kPhase0Keys), sv1);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) sv1[i] = __uint_as_float(t16[i]);
        }
      }
      // O is stable once PV(j-1, phase 1) has completed (waited on every tile)
      if (j > 0) {
        if (!__all_sync(kFull, wait_bar(bars.o_done, ph ^ 1u, p, abort_flag))) {
          return false;
        }
        tc_fence_after();
      }
      float alpha = 1.0f;
      if (__any_sync(kFull, o_rescale)) {
        alpha = o_rescale ? ex2(m_old - m) : 1.0f;
        rescale_o(alpha);
      }
      l = l * alpha + lt;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full);  // one arrival per softmax warp

      // ---------------- phase 1: keys 48..63 (same max), P to shared memory
      {
        // PV(j-1, phase 1) read the previous contents: complete (o_done above)
        uint32_t pk[8];
        lt = kGeneral ? probs16_general(sv1, bm, kPhase0Keys, m, scale, tq, p, pk)
                      : probs16_fast(sv1, fast_offset(bm, kPhase0Keys, m), scale, pk);
        *reinterpret_cast<uint4*>(ph1_row + (0u ^ ph1_swz)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(ph1_row + (16u ^ ph1_swz)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      l += lt;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full + 1);
      return true;
    };
    int j = 0;
    for (; ok && j < n_fast_tiles; ++j) ok = tile(j, std::false_type{});
    for (; ok && j < n_tiles; ++j) ok = tile(j, std::true_type{});
    // ---------------------------------------------------------- epilogue
    bool fin = __all_sync(kFull, ok) && n_tiles > 0;
    // total row sum, in the slot the last tile's exchange did not use
    if (fin) {
      const int slot = n_xchg & 1u;
      red[(slot * 2 + part) * 128 + r] = l;
      mbar_arrive(xbar);
      fin = wait_bar(xbar, n_xchg & 1u, p, abort_flag);
      if (fin) l += red[(slot * 2 + (part ^ 1)) * 128 + r];
      if (fin) fin = wait_bar(bars.o_final, 0, p, abort_flag);
    }
    if (__all_sync(kFull, fin)) {
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      uint16_t* orow = p.o + ((size_t)head * p.S + (row_valid ? qrow : 0)) * D + part * kOCols;
#pragma unroll
      for (int c = 0; c < kOCols / 32; ++c) {
        uint32_t tmp[32];
        __syncwarp();
        tmem_ld32(t_o + c * 32, tmp);
        tmem_wait_ld();
        uint32_t outw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          outw[i] = pack_bf16(__uint_as_float(tmp[2 * i]) * inv_l, __uint_as_float(tmp[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
        }
      }
      if (row_valid && part == 0 && p.lse != nullptr) p.lse[(size_t)head * p.S + qrow] = (m + __log2f(l)) * kLn2;
    }
    // a step left early on a give-up may still have TMEM accesses in flight:
    // they complete before the allocation is released
    tmem_wait_st();
    tmem_wait_ld();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

int attn_smem_bytes(int d, int n_blocks, bool qk8) {
  if (qk8) return Layout<128, true>::host_bytes(n_blocks);
  return d == 64 ? Layout<64, false>::host_bytes(n_blocks) : Layout<128, false>::host_bytes(n_blocks);
}

namespace {
template <int D, bool kQK8>
cudaError_t launch_attn_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                          int n_ctas, cudaStream_t stream) {
  const int smem = Layout<D, kQK8>::host_bytes(p.n_blocks);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, kQK8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_kernel<D, kQK8><<<n_ctas, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnParams& p, int n_ctas, cudaStream_t stream, bool qk8) {
  if (qk8) return p.d == 128 ? launch_attn_t<128, true>(tq, tk, tv, p, n_ctas, stream) : cudaErrorInvalidValue;
  return p.d == 64 ? launch_attn_t<64, false>(tq, tk, tv, p, n_ctas, stream)
                   : launch_attn_t<128, false>(tq, tk, tv, p, n_ctas, stream);
}

}  // namespace h3
