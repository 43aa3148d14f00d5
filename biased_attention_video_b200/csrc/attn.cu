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
// blocks' key lists one 64-row key block per step; each query row masks the
// key blocks its own query block does not attend, and a softmax warp whose
// query block skips a key block writes zero probabilities for it without
// reading its scores.
//
// Two CTAs share an SM (256 TMEM columns and about 100 KB of shared memory
// each), so one CTA's tensor-core work overlaps the other's softmax.
//
// A second instantiation (kQK8) takes Q and K as int8 codes with per-token
// scales: the S products run as int8 MMAs, everything else is shared.
//
// Warp roles (192 threads):
//   warps 0..3  softmax: one thread per query row (= TMEM lane); warp w owns
//               TMEM lanes [32 w, 32 w + 32), so rows 0..63 (block A) sit in
//               warps 0-1 and rows 64..127 (block B) in warps 2-3
//   warp 4      TMA producer: Q tile once, then K and V per key block (two
//               stages each)
//   warp 5      TMEM owner + single-thread tcgen05.mma issuer
//
// TMEM: S[0] [0,64), S[1] [64,128): fp32 scores of the steps j with j % 2 = 0,
// 1; O [128, 128 + d).  The bf16 probabilities of step j go back over the
// first 32 columns of S[j % 2] (TS-form PV).
//
// MMA issue order: S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...  S(j+1) is
// already computed while the softmax works on step j, so the softmax runs its
// steps back to back while the tensor cores run PV(j) and S(j+2).  The
// tcgen05.mma ops of one thread run in issue order: S(j+2) never overwrites
// P(j) before PV(j) has read it, and when the commit after S(j) fires, PV(j-2)
// has completed.  O may still be accumulating PV(j-1) while the softmax of
// step j runs, so a rescale of O first waits for PV(j-1).  Every thread owns
// its whole row, so the running max and the row sum need no exchange.
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

constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kStepKeys = 64;  // one key block per step
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 128;  // O column offset

template <int D, bool kQK8>
struct Layout {
  static constexpr int kHalves = D / 64;   // 128-byte swizzle atoms along d (bf16 V)
  static constexpr int kQAtom = 128 * 128;  // one 128-byte-wide column of the 128-row Q tile
  static constexpr int kKVAtom = 64 * 128;  // one 128-byte-wide column of a 64-row K or V block
  // Q and K: bf16, or int8 codes (one 128-byte atom holds d = 128)
  static constexpr int kQKHalves = kQK8 ? D / 128 : D / 64;
  static constexpr int kQKElems = kQK8 ? 128 : 64;  // elements per 128-byte atom
  static constexpr int kQBytes = kQKHalves * kQAtom;
  static constexpr int kKStage = kQKHalves * kKVAtom;
  static constexpr int kVStage = kHalves * kKVAtom;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;       // two stages
  static constexpr int kV = kK + 2 * kKStage;   // two stages
  static constexpr int kBars = kV + 2 * kVStage;
  // q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done, o_final, drain
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBars + kNumBars * 8;  // tmem base, abort flag, n_entries, n_fast
  static constexpr int kLists = kMisc + 16;           // bitmap A, bitmap B, key-block list
  static int host_bytes(int n_blocks) {
    const int nwords = (n_blocks + 31) / 32;
    return 1024 /*alignment slack*/ + kLists + 2 * nwords * 4 + ((n_blocks * 2 + 15) & ~15);
  }
};

struct Bars {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done, *o_final, *drain;
};

// k_full[s] / k_empty[s], v_full[s] / v_empty[s]: stage s of K / V (steps j
// with j % 2 = s).  s_full[b]: S of a step into buffer b complete (and with
// it every earlier MMA).  p_full[b]: the four softmax warps wrote the
// probabilities of a step into buffer b -- one barrier per buffer, because a
// warp may finish step j+1 (whose scores are already there) before another
// has finished step j; it can never get two steps ahead, since S(j+2) waits
// for PV(j).  o_done: PV(j) complete (one completion per step).
__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  return Bars{b, b + 1, b + 3, b + 5, b + 7, b + 9, b + 11, b + 13, b + 14, b + 15};
}

// Wait for an outstanding tcgen05.ld, with the loaded registers tied to the
// wait so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_dep(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
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
  uint32_t* bm_a = reinterpret_cast<uint32_t*>(smem + L::kLists);
  uint32_t* bm_b = bm_a + nwords;
  // entry = key block (14 bits) | attended by block A << 14 | attended by block B << 15
  uint16_t* list = reinterpret_cast<uint16_t*>(bm_b + nwords);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // Tile order: the dense (prefix) query tiles of every head first -- they
  // walk every key block, so the longest tiles start earliest and none is left
  // running alone at the end -- then the paired tiles head-major, so the ~300
  // CTAs resident at a time share one or two heads' K/V in L2.
  const int n_dense_all = p.H * p.n_dense_tiles;
  int head, qtile;
  if ((int)blockIdx.x < n_dense_all) {
    head = (int)blockIdx.x / p.n_dense_tiles;
    qtile = (int)blockIdx.x % p.n_dense_tiles;
  } else {
    const int b = (int)blockIdx.x - n_dense_all;
    head = b / p.n_paired_tiles;
    qtile = p.n_dense_tiles + b % p.n_paired_tiles;
  }
  // An earlier CTA that gave up leaves the status word set: skip the work
  // (decided once per CTA so that every thread leaves together).
  if (tid == 0) *abort_flag = *reinterpret_cast<volatile int*>(p.status) == kStatusTimeout ? 1 : 0;
  __syncthreads();
  if (*abort_flag) return;
  __syncthreads();

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars.k_full + s, 1);
      mbar_init(bars.k_empty + s, 1);
      mbar_init(bars.v_full + s, 1);
      mbar_init(bars.v_empty + s, 1);
      mbar_init(bars.s_full + s, 1);
      mbar_init(bars.p_full + s, 4);
    }
    mbar_init(bars.o_done, 1);
    mbar_init(bars.o_final, 1);
    mbar_init(bars.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
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
  if (warp == kProducerWarp) {
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
  const int n_steps = *n_entries_slot;
  const int n_fast = *n_fast_slot;  // steps whose key block takes the fast path

  if (warp == kProducerWarp) {
    if (lane == 0 && n_steps > 0) {
      // ---------------------------------------------------------- producer
      uint32_t issued_k[2] = {0u, 0u}, issued_v[2] = {0u, 0u};
      const int oob_row = p.n_blocks * 64;  // a whole block past S: zero-filled by TMA
      const int qa_row = has_a ? qb_a * 64 : oob_row, qb_row = has_b ? qb_b * 64 : oob_row;
      uint8_t* sq = smem + L::kQ;
      mbar_arrive_expect_tx(bars.q_full, L::kQBytes);
#pragma unroll
      for (int c = 0; c < L::kQKHalves; ++c) {
        tma_load_3d(sq + c * L::kQAtom, &tm_q, bars.q_full, c * L::kQKElems, qa_row, head);
        tma_load_3d(sq + c * L::kQAtom + 8192, &tm_q, bars.q_full, c * L::kQKElems, qb_row, head);
      }
      for (int j = 0; j < n_steps; ++j) {
        const int s = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const int row = (int)(list[j] & 0x3FFFu) * 64;
        uint8_t* sk = smem + L::kK + s * L::kKStage;
        uint8_t* sv = smem + L::kV + s * L::kVStage;
        if (!wait_bar(bars.k_empty + s, ph ^ 1u, p, abort_flag)) break;
        mbar_arrive_expect_tx(bars.k_full + s, L::kKStage);
#pragma unroll
        for (int c = 0; c < L::kQKHalves; ++c)
          tma_load_3d(sk + c * L::kKVAtom, &tm_k, bars.k_full + s, c * L::kQKElems, row, head);
        ++issued_k[s];
        if (!wait_bar(bars.v_empty + s, ph ^ 1u, p, abort_flag)) break;
        mbar_arrive_expect_tx(bars.v_full + s, L::kVStage);
#pragma unroll
        for (int c = 0; c < L::kHalves; ++c)
          tma_load_3d(sv + c * L::kKVAtom, &tm_v, bars.v_full + s, c * 64, row, head);
        ++issued_v[s];
      }
      // drain: every issued load must land before the CTA may exit
      drain_wait(bars.q_full, 0, p);
      for (int s = 0; s < 2; ++s) {
        if (issued_k[s]) drain_wait(bars.k_full + s, (issued_k[s] - 1) & 1u, p);
        if (issued_v[s]) drain_wait(bars.v_full + s, (issued_v[s] - 1) & 1u, p);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && n_steps > 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescS = kQK8 ? idesc_s8_s32(128, kStepKeys) : idesc_bf16_f32(128, kStepKeys, 0, 0);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      const uint32_t o_tmem = tmem_base + kTmemO;
      // S(j) = Q K(j)^T into S[j % 2]; then s_full[j % 2] and k_empty[j % 2]
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!wait_bar(bars.k_full + s, (uint32_t)(j >> 1) & 1u, p, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(kStepKeys * s);
        const uint32_t kst = k_addr + (uint32_t)(s * L::kKStage);
        // one MMA per 32-byte K step: 16 bf16 or 32 int8 elements of d
#pragma unroll
        for (int kk = 0; kk < L::kQKHalves * 4; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t adesc = sw128_desc(q_addr + c * L::kQAtom + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(kst + c * L::kKVAtom + off, 16, 1024);
          if constexpr (kQK8)
            umma_ss_i8(d_tmem, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
          else
            umma_ss(d_tmem, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bars.s_full + s);
        umma_commit(bars.k_empty + s);
        return true;
      };
      bool ok = wait_bar(bars.q_full, 0, p, abort_flag) && issue_s(0);
      if (ok && n_steps > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_steps; ++j) {
        const int s = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        if (!wait_bar(bars.p_full + s, ph, p, abort_flag) || !wait_bar(bars.v_full + s, ph, p, abort_flag)) break;
        tc_fence_after();
        // O += P(j) V(j): P at S[s] columns [0,32) (two bf16 keys per column),
        // 16 keys (2 KB of each V atom) per MMA; V read MN-major
        const uint32_t p_tmem = tmem_base + (uint32_t)(kStepKeys * s);
        const uint32_t vst = v_addr + (uint32_t)(s * L::kVStage);
#pragma unroll
        for (int kk = 0; kk < kStepKeys / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(vst + kk * 2048, L::kKVAtom, 1024);
          umma_ts(o_tmem, p_tmem + 8 * kk, bdesc, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bars.v_empty + s);
        umma_commit(bars.o_done);
        if (j + 2 < n_steps) ok = issue_s(j + 2);
      }
      umma_commit(bars.o_final);
      // drain: all issued MMAs complete before TMEM is released
      umma_commit(bars.drain);
      drain_wait(bars.drain, 0, p);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // One thread per query row: warp w handles TMEM lanes [32 w, 32 w + 32).
    // tcgen05.ld/st are warp-collective (.sync.aligned): every branch that
    // guards one is warp-uniform (a vote, or a value that is the same for the
    // whole warp).
    const int r = warp * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const uint32_t t_o = tmem_base + lane_addr + kTmemO;
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
    float l = 0.0f;       // row sum
    bool ok = n_steps > 0;

    // O *= alpha for this thread's row (warp-uniform call)
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t tmp[32];
        __syncwarp();
        tmem_ld32(t_o + c * 32, tmp);
        tmem_wait_ld_dep(tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) tmp[i] = __float_as_uint(__uint_as_float(tmp[i]) * alpha);
        tmem_st32(t_o + c * 32, tmp);
      }
    };
    auto block_mode = [&](uint32_t ent, bool attended, const uint4& kd) -> BlockMode {
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
      return bm;
    };
    // the list entry and key-block descriptor of a step, fetched one step
    // ahead so that the descriptor load overlaps the previous step
    struct Ahead {
      uint32_t e;
      uint4 kd;
    };
    auto fetch = [&](int j) -> Ahead {
      Ahead a{0u, make_uint4(0u, 0u, 0u, 0u)};
      if (j < n_steps) {
        a.e = list[j];
        if ((a.e >> my_bit) & 1u) a.kd = __ldg(p.kv_desc + (a.e & 0x3FFFu));
      }
      return a;
    };

    Ahead cur = fetch(0);
    // One key step; kGeneral selects the per-key path (validity, per-key
    // penalty) that the few slow key blocks need, kept out of the loop over
    // the others.  A warp's 32 rows belong to one query block, so whether it
    // attends the step's key block is warp-uniform.
    auto step = [&](int j, auto general) -> bool {
      constexpr bool kGeneral = decltype(general)::value;
      const int s = j & 1;
      const bool att = ((cur.e >> my_bit) & 1u) != 0u;
      const BlockMode bm = block_mode(cur.e, att, cur.kd);
      cur = fetch(j + 1);
      if (!__all_sync(kFull, wait_bar(bars.s_full + s, (uint32_t)(j >> 1) & 1u, p, abort_flag))) return false;
      tc_fence_after();
      const uint32_t t_s = tmem_base + lane_addr + (uint32_t)(kStepKeys * s);
      float sv[64];
      float pmax = -INFINITY;
      if (att) {
        uint32_t u[32], w[32];
        __syncwarp();
        tmem_ld32(t_s, u);
        tmem_ld32(t_s + 32, w);
        tmem_wait_ld_dep(u);
        tmem_wait_ld_dep(w);
        if constexpr (kQK8) {
          const float* ks = p.k_scale + ((size_t)head * p.scale_stride + bm.key0);
          qk8_scores<32>(u, ks, sv);
          qk8_scores<32>(w, ks + 32, sv + 32);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            sv[i] = __uint_as_float(u[i]);
            sv[32 + i] = __uint_as_float(w[i]);
          }
        }
        pmax = kGeneral ? part_max<64>(sv, bm, 0) : full_max<64>(sv, bm);
      }
      const float mx = pmax * scale;
      // Conditional rescale: the running max only moves when it grows by more
      // than 2^8; below that the stale max keeps every probability <= 256.
      const bool grow = mx > m + kRescaleThreshold;
      const bool o_rescale = grow && m > -INFINITY;
      const float m_old = m;
      if (grow) m = mx;
      if (__any_sync(kFull, o_rescale)) {
        // O may still be accumulating PV(j-1): wait for it first
        if (!__all_sync(kFull, wait_bar(bars.o_done, (uint32_t)(j - 1) & 1u, p, abort_flag))) return false;
        tc_fence_after();
        const float alpha = o_rescale ? ex2(m_old - m) : 1.0f;
        rescale_o(alpha);
        l *= alpha;
      }
      uint32_t pk[32];
      if (att) {
        float lt = 0.0f;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          lt += kGeneral ? probs16_general(sv + 16 * g, bm, 16 * g, m, scale, tq, p, pk + 8 * g)
                         : probs16_fast(sv + 16 * g, fast_offset(bm, 16 * g, m), scale, pk + 8 * g);
        l += lt;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }
      __syncwarp();
      tmem_st32(t_s, pk);  // P over the step's first 32 score columns
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full + s);  // one arrival per softmax warp
      return true;
    };

    int j = 0;
    for (; ok && j < n_fast; ++j) ok = step(j, std::false_type{});
    for (; ok && j < n_steps; ++j) ok = step(j, std::true_type{});
    // ---------------------------------------------------------- epilogue
    bool fin = __all_sync(kFull, ok) && n_steps > 0;
    if (fin) fin = __all_sync(kFull, wait_bar(bars.o_final, 0, p, abort_flag));
    if (fin) {
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      uint16_t* orow = p.o + ((size_t)head * p.S + (row_valid ? qrow : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t tmp[32];
        __syncwarp();
        tmem_ld32(t_o + c * 32, tmp);
        tmem_wait_ld_dep(tmp);
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
      if (row_valid && p.lse != nullptr) p.lse[(size_t)head * p.S + qrow] = (m + __log2f(l)) * kLn2;
    }
    // a step left early on a give-up may still have TMEM accesses in flight:
    // they complete before the allocation is released
    tmem_wait_st();
    tmem_wait_ld();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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
