// Device helpers shared by the attention kernels: key masks and the online
// softmax step of one query row over one 128-key tile.
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

// ---------------------------------------------------------------- packed fp32
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair, x <= 8, on the FMA pipe instead of the special-function
// unit.  Range reduction x = j + f with j = round-to-nearest(x) (by adding
// 1.5 * 2^23), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose
// coefficients we fitted to minimise the maximum relative error on
// [-1/2, 1/2] (7.5e-5 in fp32 Horner form, far below the bf16 rounding the
// result receives next); j is added to the exponent field.  Inputs below
// -125 are clamped there (2^-125 ~ 2.4e-38), so callers must not pass -inf
// for keys that have to contribute exactly zero.
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& y0, float& y1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = fadd2(x, f2(kRound, kRound));                // 2^23*1.5 + j (exact)
  const uint64_t j = fadd2(t, f2(-kRound, -kRound));              // j as float
  const uint64_t f = ffma2(j, f2(-1.f, -1.f), x);                 // x - j
  uint64_t p = ffma2(f2(0x1.c3f6fep-5f, 0x1.c3f6fep-5f), f, f2(0x1.f0ddfep-3f, 0x1.f0ddfep-3f));
  p = ffma2(p, f, f2(0x1.62f31ap-1f, 0x1.62f31ap-1f));
  p = ffma2(p, f, f2(0x1.fff692p-1f, 0x1.fff692p-1f));
  float p0, p1, t0, t1;
  unf2(p, p0, p1);
  unf2(t, t0, t1);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Running state of one query row: max of the scores seen (raw q.k units; the
// exponent base is fixed only when the max grows by more than `thr`) and the
// sum of the probabilities relative to it.
struct RowState {
  float m = -INFINITY;
  float l = 0.f;
};

// One online-softmax step over a 128-key tile.  s: the row's raw scores
// (masked keys become -inf); vm: keys allowed.  Writes P = 2^(s*sl2 - m*sl2)
// as packed bf16 pairs, adds their sum to st.l, and returns true when the
// row's reference max moved (then O must be multiplied by *corr).  Scaling
// and summing use packed fp32x2 arithmetic; when every key of the tile is
// allowed, one pair in four is exponentiated on the FMA pipe
// (exp2_poly_pair) and the rest on the special-function unit, which would
// otherwise be the busiest unit of the softmax.
__device__ __forceinline__ bool softmax_tile(float (&s)[128], const uint32_t (&vm)[4], RowState& st,
                                             float sl2, float thr, uint32_t (&pk)[64],
                                             float& corr) {
  const bool full = (vm[0] & vm[1] & vm[2] & vm[3]) == kFullMask;
  if (!full) {
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!((vm[w] >> i) & 1u)) s[w * 32 + i] = -INFINITY;
  }
  // row max: 8 independent chains of 3-input max, then a small tree
  float m8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m8[c] = fmax3f(s[c], s[c + 8], s[c + 16]);
#pragma unroll
  for (int i = 24; i < 120; i += 16)
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = fmax3f(m8[c], s[i + c], s[i + 8 + c]);
#pragma unroll
  for (int c = 0; c < 8; ++c) m8[c] = fmaxf(m8[c], s[120 + c]);
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
  const uint64_t scale2 = f2(sl2, sl2), neg_ms2 = f2(-ms, -ms);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial sums
  if (full) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      float x0, x1, p0, p1;
      unf2(ffma2(f2(s[2 * i], s[2 * i + 1]), scale2, neg_ms2), x0, x1);
      if ((i & 3) == 3) {
        exp2_poly_pair(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      float x0, x1;
      unf2(ffma2(f2(s[2 * i], s[2 * i + 1]), scale2, neg_ms2), x0, x1);
      const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  }
  const uint64_t a = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  float a0, a1;
  unf2(a, a0, a1);
  st.l += a0 + a1;
  return need;
}

// Multiply `ncols` fp32 accumulator columns of this thread's TMEM lane by f.
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

namespace bsa {

// One online-softmax step over a 64-key half tile (see softmax_tile).  When
// every key of the half is allowed, one pair in four is exponentiated on the
// FMA pipe (exp2_poly_pair) and the rest on the special-function unit, which
// would otherwise be the busiest unit of the softmax.
__device__ __forceinline__ bool softmax_half(float (&s)[64], const uint32_t (&vm)[2], RowState& st,
                                             float sl2, float thr, uint32_t (&pk)[32],
                                             float& corr) {
  const bool full = (vm[0] & vm[1]) == kFullMask;
  if (!full) {
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!((vm[w] >> i) & 1u)) s[w * 32 + i] = -INFINITY;
  }
  float m4[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) m4[c] = fmax3f(s[c], s[c + 4], s[c + 8]);
#pragma unroll
  for (int i = 12; i < 60; i += 8)
#pragma unroll
    for (int c = 0; c < 4; ++c) m4[c] = fmax3f(m4[c], s[i + c], s[i + 4 + c]);
#pragma unroll
  for (int c = 0; c < 4; ++c) m4[c] = fmaxf(m4[c], s[60 + c]);
  const float mx = fmax3f(m4[0], m4[1], fmaxf(m4[2], m4[3]));
  const float m_new = fmaxf(st.m, mx);
  const bool need = m_new > st.m + thr;
  corr = 1.f;
  if (need) {
    corr = ex2_approx((st.m - m_new) * sl2);
    st.m = m_new;
    st.l *= corr;
  }
  const float ms = (st.m == -INFINITY) ? 0.f : st.m * sl2;
  const uint64_t scale2 = f2(sl2, sl2), neg_ms2 = f2(-ms, -ms);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial sums
  if (full) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float x0, x1, p0, p1;
      unf2(ffma2(f2(s[2 * i], s[2 * i + 1]), scale2, neg_ms2), x0, x1);
      if ((i & 3) == 3) {
        exp2_poly_pair(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float x0, x1;
      unf2(ffma2(f2(s[2 * i], s[2 * i + 1]), scale2, neg_ms2), x0, x1);
      const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  }
  const uint64_t a = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  float a0, a1;
  unf2(a, a0, a1);
  st.l += a0 + a1;
  return need;
}

// 32 lanes x 64 columns of 32-bit from tensor memory (two loads, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
  uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(lo[0]), "=r"(lo[1]), "=r"(lo[2]), "=r"(lo[3]), "=r"(lo[4]), "=r"(lo[5]), "=r"(lo[6]),
        "=r"(lo[7]), "=r"(lo[8]), "=r"(lo[9]), "=r"(lo[10]), "=r"(lo[11]), "=r"(lo[12]),
        "=r"(lo[13]), "=r"(lo[14]), "=r"(lo[15]), "=r"(lo[16]), "=r"(lo[17]), "=r"(lo[18]),
        "=r"(lo[19]), "=r"(lo[20]), "=r"(lo[21]), "=r"(lo[22]), "=r"(lo[23]), "=r"(lo[24]),
        "=r"(lo[25]), "=r"(lo[26]), "=r"(lo[27]), "=r"(lo[28]), "=r"(lo[29]), "=r"(lo[30]),
        "=r"(lo[31]), "=r"(hi[0]), "=r"(hi[1]), "=r"(hi[2]), "=r"(hi[3]), "=r"(hi[4]), "=r"(hi[5]),
        "=r"(hi[6]), "=r"(hi[7]), "=r"(hi[8]), "=r"(hi[9]), "=r"(hi[10]), "=r"(hi[11]),
        "=r"(hi[12]), "=r"(hi[13]), "=r"(hi[14]), "=r"(hi[15]), "=r"(hi[16]), "=r"(hi[17]),
        "=r"(hi[18]), "=r"(hi[19]), "=r"(hi[20]), "=r"(hi[21]), "=r"(hi[22]), "=r"(hi[23]),
        "=r"(hi[24]), "=r"(hi[25]), "=r"(hi[26]), "=r"(hi[27]), "=r"(hi[28]), "=r"(hi[29]),
        "=r"(hi[30]), "=r"(hi[31])
      : "r"(taddr), "r"(taddr + 32)
      : "memory");
}

}  // namespace bsa
