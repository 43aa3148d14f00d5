// Softmax-side helpers shared by the attention kernels: bounded mbarrier
// waits with a CTA-wide abort flag, the temporal penalty in log2 units
// ("Flash Partitions for H3 native temporal alignment", section 1:
// penalty(dt) = min(strength (max(dt - window, 0) / falloff)^2, cap)), and the
// per-16-key probability blocks of the online softmax.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fastmath.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace h3 {
namespace sm {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ float ex2(float x) { return ex2_mufu(x); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void report(int* status, int code) { atomicCAS(status, 0, code); }

// Bounded wait with CTA-wide abort.  On give-up: raise the CTA abort flag and
// the global status word.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const AttnParams& p,
                                         volatile int* abort) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    bool give_up = i >= p.wait_polls;
    if ((i & 1023u) == 1023u) {
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      give_up = give_up || now - t0 > p.wait_ns;
    }
    if (give_up) {
      *abort = 1;
      report(p.status, kStatusTimeout);
      return false;
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

__device__ __forceinline__ float block_penalty_log2(float tq, float tk, const AttnParams& p) {
  const float dt = fabsf(tq - tk);
  const float ex = fmaxf(dt - p.window, 0.0f) * p.inv_falloff;
  return fminf(p.strength_log2 * ex * ex, p.cap_log2);
}

// How a row treats its key block in the current tile:
//   mode 0  skip (the row's query block does not attend the block)
//   mode 1  attended, no penalty
//   mode 2  attended, penalty pen_a on keys [0, split) and pen_b on [split, 64)
//           (log2 units; a block whose guide keys share one time, or two
//           contiguous runs of guide / other keys)
//   mode 3  attended, per-key penalty from the keys' guide times
struct BlockMode {
  int mode, nv, key0, split;  // nv: valid keys; key0: first key (sequence row)
  float pen_a, pen_b;
};

// Probabilities of 16 keys [c0, c0 + 16) of the thread's block, given the row
// max m (log2 units), as 8 bf16 pairs; they return their fp32 sum.
//
// Common case (every lane of the warp): modes 0 to 2 with all 16 keys valid.
// The offset is -(m + constant penalty), or -inf for a block the row does not
// attend (2^-inf = 0), so the three modes share one branch-free path; pairs are
// scaled and offset by one f32x2 FMA and exponentiated on MUFU.
__device__ __forceinline__ float probs16_fast(const float* s, float off, float scale, uint32_t* pk) {
  const uint64_t scale2 = f2_pack(scale, scale), off2 = f2_pack(off, off);
  uint64_t acc2[2] = {f2_pack(0.0f, 0.0f), f2_pack(0.0f, 0.0f)};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a, b;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), scale2, off2), a, b);
    a = ex2(a);
    b = ex2(b);
    acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(a, b));
    pk[i] = pack_bf16(a, b);
  }
  float a0, a1, b0, b1;
  f2_unpack(acc2[0], a0, a1);
  f2_unpack(acc2[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// General case (rare: a block with per-key penalties -- guide keys of several
// times, or guide and other keys mixed -- or the partial last block): each of
// the 16 keys with its own validity and penalty.  A key's guide time comes from
// gtime (NaN for a key that is not a guide key: the penalty formula then gives
// max(NaN - window, 0) = 0), read as four broadcast 16-byte loads.
__device__ __forceinline__ float probs16_general(const float* s, const BlockMode& bm, int c0, float m, float scale,
                                                 float tq, const AttnParams& p, uint32_t* pk) {
  float lt = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // four keys at a time keeps few values live
    float pen[4];
    if (bm.mode == 3) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(p.gtime + bm.key0 + c0) + q);
      pen[0] = block_penalty_log2(tq, t.x, p);
      pen[1] = block_penalty_log2(tq, t.y, p);
      pen[2] = block_penalty_log2(tq, t.z, p);
      pen[3] = block_penalty_log2(tq, t.w, p);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) pen[e] = c0 + 4 * q + e < bm.split ? bm.pen_a : bm.pen_b;
    }
    float pp[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = c0 + 4 * q + e;
      pp[e] = (bm.mode != 0 && col < bm.nv) ? ex2(fmaf(s[4 * q + e], scale, -(m + pen[e]))) : 0.0f;
    }
    lt += (pp[0] + pp[1]) + (pp[2] + pp[3]);
    pk[2 * q] = pack_bf16(pp[0], pp[1]);
    pk[2 * q + 1] = pack_bf16(pp[2], pp[3]);
  }
  return lt;
}

// Offset of a 16-key group on the fast path: -inf for a block the row does
// not attend, else -(m + the group's penalty) (a fast block's penalty runs
// split on a group boundary).
__device__ __forceinline__ float fast_offset(const BlockMode& bm, int c0, float m) {
  return bm.mode == 0 ? -INFINITY : -(m + (c0 < bm.split ? bm.pen_a : bm.pen_b));
}

// Int8 QK: N raw s32 scores (exact integer dot products of the codes, |s| <
// 2^22 for d = 128) to fp32 by the exponent trick (2^23 + 2^22 + s is exact
// in fp32, and its bits are those of the integer plus a constant), times the
// keys' scales ks[0..N) (16-byte aligned).
template <int N>
__device__ __forceinline__ void qk8_scores(const uint32_t* raw, const float* ks, float* out) {
  constexpr int kMagicBits = 0x4B400000;     // 12582912.0f = 2^23 + 2^22
  const uint64_t magic2 = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 s = __ldg(reinterpret_cast<const float4*>(ks + i));
    const uint64_t a = f2_mul(f2_sub(f2_pack(__int_as_float((int)raw[i] + kMagicBits),
                                             __int_as_float((int)raw[i + 1] + kMagicBits)), magic2),
                              f2_pack(s.x, s.y));
    const uint64_t b = f2_mul(f2_sub(f2_pack(__int_as_float((int)raw[i + 2] + kMagicBits),
                                             __int_as_float((int)raw[i + 3] + kMagicBits)), magic2),
                              f2_pack(s.z, s.w));
    f2_unpack(a, out[i], out[i + 1]);
    f2_unpack(b, out[i + 2], out[i + 3]);
  }
}

// Maximum over N keys of a fully valid block (-inf if the row skips it).
template <int N>
__device__ __forceinline__ float full_max(const float* s, const BlockMode& bm) {
  float mp[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) mp[a] = fmaxf(s[a], s[a + 4]);
#pragma unroll
  for (int i = 8; i < N; i += 8)
#pragma unroll
    for (int a = 0; a < 4; ++a) mp[a] = max3f(mp[a], s[i + a], s[i + 4 + a]);
  return bm.mode == 0 ? -INFINITY : fmaxf(max3f(mp[0], mp[1], mp[2]), mp[3]);
}

// Maximum over the valid keys [c0, c0 + N) of the thread's block (-inf if none).
template <int N>
__device__ __forceinline__ float part_max(const float* s, const BlockMode& bm, int c0) {
  float pmax = -INFINITY;
  if (bm.mode != 0) {
    if (bm.nv >= c0 + N) {
      float mp[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) mp[a] = fmaxf(s[a], s[a + 4]);
#pragma unroll
      for (int i = 8; i < N; i += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a) mp[a] = max3f(mp[a], s[i + a], s[i + 4 + a]);
      pmax = fmaxf(max3f(mp[0], mp[1], mp[2]), mp[3]);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i)
        if (c0 + i < bm.nv) pmax = fmaxf(pmax, s[i]);
    }
  }
  return pmax;
}

}  // namespace sm
}  // namespace h3
