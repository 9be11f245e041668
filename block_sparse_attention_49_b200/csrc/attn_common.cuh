// Device helpers shared by the attention kernels: key masks and the online
// softmax step of one query row over one tile of keys.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace bsa {

constexpr uint32_t kFullMask = 0xffffffffu;

// Set bits [lo, hi) of a 128-bit mask (0 <= lo <= hi <= 128).
__device__ __forceinline__ void set_range(uint32_t (&m)[4], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int a = max(lo, 32 * w), b = min(hi, 32 * w + 32);
    if (b > a) {
      const int n = b - a;
      m[w] |= (n == 32 ? kFullMask : ((1u << n) - 1u)) << (a - 32 * w);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Running state of one query row: max of the scores seen (raw q.k units; the
// exponent base is fixed only when the max grows by more than `thr`) and the
// sum of the probabilities relative to it.
struct RowState {
  float m = -INFINITY;
  float l = 0.f;
};

// First half of an online-softmax step over NC keys (NC = 64 or 128): mask
// the keys not allowed (vm) to -inf, take the row max and decide whether the
// row's reference max moves (it does only when the max grows by more than
// `thr`, so P stays below 2^(thr*sl2)).  On a move st.m and st.l are updated
// and *corr is the factor O must be multiplied by.  *ms2 receives the packed
// pair (-m*sl2, -m*sl2) for softmax_exp.  MASK = false: the caller knows
// every key is allowed, and the masking code is left out altogether.
template <int NC, bool MASK = true>
__device__ __forceinline__ bool softmax_max(float (&s)[NC], const uint32_t (&vm)[NC / 32],
                                            RowState& st, float sl2, float thr, float& corr,
                                            uint64_t& neg_ms2) {
  static_assert(NC == 64 || NC == 128, "column count");
  uint32_t all = kFullMask;
#pragma unroll
  for (int w = 0; w < NC / 32; ++w) all &= vm[w];
  if (MASK && all != kFullMask) {
#pragma unroll
    for (int w = 0; w < NC / 32; ++w)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!((vm[w] >> i) & 1u)) s[w * 32 + i] = -INFINITY;
  }
  // row max: 8 independent chains of 3-input max, then a small tree
  float m8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m8[c] = s[c];
  constexpr int kTail = 8 + ((NC - 8) / 16) * 16;
#pragma unroll
  for (int i = 8; i + 16 <= NC; i += 16)
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = fmax3f(m8[c], s[i + c], s[i + 8 + c]);
  if constexpr (kTail < NC) {
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = fmaxf(m8[c], s[kTail + c]);
  }
  const float mx = fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]),
                          fmaxf(m8[6], m8[7]));
  const float m_new = fmaxf(st.m, mx);
  const bool need = m_new > st.m + thr;
  corr = 1.f;
  if (need) {
    corr = ex2_approx((st.m - m_new) * sl2);
    st.m = m_new;
    st.l *= corr;
  }
  const float ms = (st.m == -INFINITY) ? 0.f : st.m * sl2;
  neg_ms2 = f2(-ms, -ms);
  return need;
}

// Second half, for keys [OFF, OFF + NK) of the row: P = 2^(s*sl2 - m*sl2)
// written as packed bf16 pairs to pk[0 .. NK/2), their sum added to the
// packed partial sums acc.  Scaling and summing use packed fp32x2
// arithmetic (half the instructions).
template <int OFF, int NK, int NC>
__device__ __forceinline__ void softmax_exp(const float (&s)[NC], float sl2, uint64_t neg_ms2,
                                            uint32_t (&pk)[NK / 2], uint64_t (&acc)[4]) {
  const uint64_t scale2 = f2(sl2, sl2);
#pragma unroll
  for (int i = 0; i < NK / 2; ++i) {
    float x0, x1;
    unf2(ffma2(f2(s[OFF + 2 * i], s[OFF + 2 * i + 1]), scale2, neg_ms2), x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
}

// Two floats to two e4m3 bytes (nearest, ties to even, saturating at +-448),
// lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// softmax_exp for 8-bit P: keys [OFF, OFF + 64) as e4m3, four to a word
// (P <= 2^8 < 448), into pk[0 .. 16); the sums take the unrounded values.
template <int OFF, int NC>
__device__ __forceinline__ void softmax_exp_e4m3(const float (&s)[NC], float sl2, uint64_t neg_ms2,
                                                 uint32_t (&pk)[16], uint64_t (&acc)[4]) {
  const uint64_t scale2 = f2(sl2, sl2);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1, x2, x3;
    unf2(ffma2(f2(s[OFF + 4 * i], s[OFF + 4 * i + 1]), scale2, neg_ms2), x0, x1);
    unf2(ffma2(f2(s[OFF + 4 * i + 2], s[OFF + 4 * i + 3]), scale2, neg_ms2), x2, x3);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
    acc[(2 * i) & 3] = fadd2(acc[(2 * i) & 3], f2(p0, p1));
    acc[(2 * i + 1) & 3] = fadd2(acc[(2 * i + 1) & 3], f2(p2, p3));
    pk[i] = pack_e4m3x2(p0, p1) | (pack_e4m3x2(p2, p3) << 16);
  }
}

// Adds the packed partial sums to the row's running sum.
__device__ __forceinline__ void softmax_sum(RowState& st, const uint64_t (&acc)[4]) {
  const uint64_t a = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  float a0, a1;
  unf2(a, a0, a1);
  st.l += a0 + a1;
}

// Multiply NCOLS fp32 accumulator columns of this thread's TMEM lane by f.
template <int NCOLS>
__device__ __forceinline__ void tmem_scale(uint32_t taddr, float f) {
#pragma unroll
  for (int c = 0; c < NCOLS / 32; ++c) {
    uint32_t o32[32];
    tmem_ld32(taddr + c * 32, o32);
#pragma unroll
    for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * f);
    tmem_st32(taddr + c * 32, o32);
  }
}

}  // namespace bsa
