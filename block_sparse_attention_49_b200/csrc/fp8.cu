// e4m3 quantization of Q, K, V for the 8-bit draft attention (Draft
// Attention article, closing paragraph: quantization as the next step; the
// article fixes no format).  One scale per (tensor, batch, head):
//   scale = fp32(max |x|) / 448 (1 when the head is all zero),
//   code  = e4m3 nearest to x / scale (fp32 division), ties to even,
//           saturating at +-448.
// Three kernels on natural-layout [B, N, Hh, D] tensors: the per-head
// maximum (one atomicMax per CTA; |x| of a float orders like its bits), the
// scales (and their fp32 reciprocals, kept in the maximum's workspace), and
// the conversion (8 values per thread, 16-byte loads).
//
// The conversion needs x / scale only to e4m3 precision, so it multiplies by
// the reciprocal r = fp32(1 / scale) and divides only where that could give
// another code.  With z = x / scale exactly, x * r carries two roundings of
// relative size at most 2^-24 and fp32(z) one, so the two fp32 numbers are at
// most 3 units in the last place apart (both in the binade of z).  Rounding to
// e4m3 (3 mantissa bits) can then differ only if a rounding boundary of e4m3
// -- the midpoint between two neighbouring codes, where the 20 fp32 mantissa
// bits below the e4m3 ones read 0x80000 -- lies within 3 units of x * r.
// Products at least 4 units from every midpoint, in e4m3's normal range
// [2^-6, 448], are used as they are; all others take the fp32 division: the
// subnormal range, and near-midpoint products, about 8 in 2^20 values when
// the quotients are not short binary fractions (a head whose maximum has a
// short mantissa, a power of two say, gives many exact quotients, and those
// that are midpoints are ties the division must settle).  The codes are those
// of the division everywhere.
#include <cuda_bf16.h>

#include <algorithm>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kTokPerCta = 512;

template <int D>
__global__ void __launch_bounds__(kThreads)
    e4m3_amax_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                     const uint4* __restrict__ v, int B, int Hh, int64_t N, int which0,
                     uint32_t* amax) {
  constexpr int kTPR = D / 8;                  // threads per token row of one head
  constexpr int kRowsPerPass = kThreads / kTPR;
  __shared__ float red[kThreads / 32];
  const int which = which0 + blockIdx.z;
  const int bh = blockIdx.y, b = bh / Hh, h = bh - b * Hh;
  const uint4* x = which == 0 ? q : (which == 1 ? k : v);
  const int64_t n0 = (int64_t)blockIdx.x * kTokPerCta;
  const int sub = threadIdx.x % kTPR;
  float m = 0.f;
  for (int r = threadIdx.x / kTPR; r < kTokPerCta; r += kRowsPerPass) {
    const int64_t n = n0 + r;
    if (n >= N) break;
    const uint4 u = __ldg(x + (((int64_t)b * N + n) * Hh + h) * (D / 8) + sub);
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(pv[e]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) t = fmaxf(t, red[w]);
    atomicMax(amax + ((int64_t)which * B + b) * Hh + h, __float_as_uint(t));
  }
}

// scale = max / 448 (1 for an all-zero head); the maximum's slot then holds
// the fp32 reciprocal of the scale for the conversion
__global__ void e4m3_scales_kernel(uint32_t* __restrict__ amax, int n, float* scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = __uint_as_float(amax[i]);
    const float sc = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
    scales[i] = sc;
    amax[i] = __float_as_uint(__frcp_rn(sc));
  }
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// x / s to the precision e4m3 keeps (r = fp32(1 / s); see the file comment)
__device__ __forceinline__ float quotient_for_e4m3(float x, float s, float r) {
  const float y = x * r;
  const uint32_t a = __float_as_uint(y) & 0x7fffffffu;
  const int d = (int)(a & 0xfffffu) - 0x80000;  // units in the last place to the midpoint
  const bool safe = a >= 0x3c800000u && a <= 0x43e00000u && (d >= 4 || d <= -4);  // [2^-6, 448]
  return safe ? y : __fdiv_rn(x, s);
}

// grid-stride over pairs of 8-value groups of one tensor (blockIdx.y): the
// two groups of a pair lie in one token row, so they share the index
// arithmetic and the scale loads, and their 16 codes go out in one 16-byte
// store (the e4m3 buffers are 16-byte aligned: the entry points check it).
// The group count of a tensor is below 2^31 (the plan checks it), so 32-bit
// indices and magic-number division give (b, h) of a group
template <int D>
__global__ void __launch_bounds__(kThreads)
    e4m3_convert_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                        const uint4* __restrict__ v, uint2* __restrict__ q8, uint2* __restrict__ k8,
                        uint2* __restrict__ v8, int B, int Hh, uint32_t per, FastDiv div_Hh,
                        FastDiv div_batch, const float* __restrict__ scales,
                        const float* __restrict__ recips) {
  constexpr int kShift = D == 128 ? 4 : 3;  // log2(D / 8)
  const int which = blockIdx.y;
  const uint4* x = which == 0 ? q : (which == 1 ? k : v);
  uint2* y = which == 0 ? q8 : (which == 1 ? k8 : v8);
  const float* sc = scales + (int64_t)which * B * Hh;
  const float* rc = recips + (int64_t)which * B * Hh;
  const uint32_t stride = gridDim.x * kThreads;
  const uint32_t per2 = per >> 1;  // pairs of groups (a row holds 8 or 16 groups)
  for (uint32_t r2 = blockIdx.x * kThreads + threadIdx.x; r2 < per2; r2 += stride) {
    const uint32_t r = r2 << 1;
    const uint32_t row = r >> kShift;                  // (b * N + n) * Hh + h
    const uint32_t bn = div_Hh.div(row);
    const int h = (int)(row - bn * (uint32_t)Hh);
    const int b = (int)div_batch.div(r);               // r / (N * Hh * D / 8)
    const float s = __ldg(sc + b * Hh + h), rs = __ldg(rc + b * Hh + h);
    const uint4 u0 = __ldg(x + r), u1 = __ldg(x + r + 1);
    uint32_t w[4];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(g ? &u1 : &u0);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 f0 = __bfloat1622float2(pv[2 * i]), f1 = __bfloat1622float2(pv[2 * i + 1]);
        w[2 * g + i] = e4m3x2(quotient_for_e4m3(f0.x, s, rs), quotient_for_e4m3(f0.y, s, rs)) |
                       (e4m3x2(quotient_for_e4m3(f1.x, s, rs), quotient_for_e4m3(f1.y, s, rs)) << 16);
      }
    }
    reinterpret_cast<uint4*>(y)[r2] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const Geometry& g, uint32_t* amax_ws, const void* q, const void* k,
                                 const void* v, void* q8, void* k8, void* v8, float* scales,
                                 cudaStream_t st, bool qk_amax_ready) {
  const int64_t N = (int64_t)g.T * g.P;
  const int nsc = 3 * g.B * g.Hh;
  cudaError_t e = cudaSuccess;
  // qk_amax_ready: the maxima of Q and K are already in amax_ws (recorded by
  // the draft pooling, which read both), so only V's are taken here
  if (!qk_amax_ready) {
    e = cudaMemsetAsync(amax_ws, 0, sizeof(uint32_t) * nsc, st);
    if (e != cudaSuccess) return e;
  }
  const int which0 = qk_amax_ready ? 2 : 0;
  const dim3 grid((unsigned)((N + kTokPerCta - 1) / kTokPerCta), (unsigned)(g.B * g.Hh),
                  (unsigned)(3 - which0));
  auto qq = reinterpret_cast<const uint4*>(q);
  auto kk = reinterpret_cast<const uint4*>(k);
  auto vv = reinterpret_cast<const uint4*>(v);
  if (g.D == 128)
    e4m3_amax_kernel<128><<<grid, kThreads, 0, st>>>(qq, kk, vv, g.B, g.Hh, N, which0, amax_ws);
  else
    e4m3_amax_kernel<64><<<grid, kThreads, 0, st>>>(qq, kk, vv, g.B, g.Hh, N, which0, amax_ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e4m3_scales_kernel<<<(nsc + 255) / 256, 256, 0, st>>>(amax_ws, nsc, scales);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t per = (int64_t)g.B * N * g.Hh * (g.D / 8);  // groups per tensor (< 2^31)
  const dim3 cgrid(
      (unsigned)std::min<int64_t>((per + kThreads - 1) / kThreads, (int64_t)sms * 8), 3);
  const FastDiv div_Hh((uint32_t)g.Hh), div_batch((uint32_t)(N * g.Hh * (g.D / 8)));
  auto y0 = reinterpret_cast<uint2*>(q8);
  auto y1 = reinterpret_cast<uint2*>(k8);
  auto y2 = reinterpret_cast<uint2*>(v8);
  if (g.D == 128)
    e4m3_convert_kernel<128><<<cgrid, kThreads, 0, st>>>(qq, kk, vv, y0, y1, y2, g.B, g.Hh,
                                                         (uint32_t)per, div_Hh, div_batch, scales,
                                                         reinterpret_cast<const float*>(amax_ws));
  else
    e4m3_convert_kernel<64><<<cgrid, kThreads, 0, st>>>(qq, kk, vv, y0, y1, y2, g.B, g.Hh,
                                                        (uint32_t)per, div_Hh, div_batch, scales,
                                                        reinterpret_cast<const float*>(amax_ws));
  return cudaGetLastError();
}

}  // namespace bsa
