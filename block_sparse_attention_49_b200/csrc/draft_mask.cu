// Draft mask (Draft Attention article: tokens reshaped to [t,h,w]; Q and K
// average-pooled over pool_h x pool_w tiles into a low-resolution draft
// attention map; the map yields a sparse mask that keeps only the important
// block connections, at a stated sparsity; pool_h*pool_w equals the block
// size of the block-sparse attention that follows).
//
// Two kernels, on the tile-layout slot tensors or in place on the natural
// layout (each block = one pool_h x pool_w tile):
//  pool:  qbar/kbar[b,h,blk,:] = mean of the tile's tokens: the sum runs
//         in fp64, sequentially over the tile's tokens in row-major order,
//         is divided once by the token count and rounded once to fp32.
//         With max pooling (which the article's authors tried before
//         settling on the average) it is the channel-wise maximum instead,
//         exact in any order.  16-byte loads, four rows ahead; HBM bound.
//  score_topk: for a group of query-block rows of one (b, head), the fp32
//         logits L[i][j] = sum_c qbar_i[c]*kbar_j[c] (sequential over c, the
//         product and the sum each rounded to fp32, no fused multiply-add),
//         then per row the k largest, ties to the lower j, by k rounds of a
//         warp-wide arg-max; written ascending.  Optionally the draft map
//         softmax_j(L[i][j]/sqrt(D)), evaluated in fp64 and stored as fp32.
// With this fixed evaluation order the selection is reproducible bit for bit
// by any implementation that follows the same order.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cfloat>
#include <type_traits>

#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kKeyChunk = 32;  // key blocks staged in shared memory per step
constexpr int kRegCand = 16;   // top-k candidates per lane held in registers (Nb <= 512)
constexpr unsigned kFullMaskScore = 0xffffffffu;

// ---------------------------------------------------------------------------
// Pooling.  One group of D/8 threads per unit (Q or K, tile, batch, head);
// each thread owns 8 channels: eight independent fp64 chains, each the
// sequential sum over the tile's tokens in row-major order, stored as fp32.  Token rows are
// read with 16-byte loads, four rows ahead of the additions.  Units are
// ordered heads fastest, so the groups of a warp read neighbouring 256-byte
// rows of one token.  At most 64 registers a thread: four 256-thread CTAs fit
// on an SM, so a 12-head Wan-1.3B-like problem runs in one wave.
//   natural layout [B, N, Hh, D]: the tokens of the pool_h x pool_w tile
//     inside the grid, row by row;
//   slot layout [B, Hh, Npad, D]: the block's non-empty slots in order (runs
//     of consecutive slots, from the plan's validity bits).
// Optionally records max |x| per (Q or K, batch, head) for the e4m3 scales.
// ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

struct PoolParams {
  int B, Hh, T, H, W, ph, pw, TH, TW, block;
  int64_t nblocks, Npad, groups_per_tensor;
  int use_max;
  const uint32_t* tile_valid;
  uint32_t* amax;  // [3][B][Hh] float bits, or null
  float* ws;
};

template <int D, bool NAT, bool MAXP, bool AMAX>
__global__ void __launch_bounds__(kPoolThreads, 4)
    draft_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const PoolParams p) {
  constexpr int kTPG = D / 8;  // threads per group
  constexpr int kAhead = 4;
  const int64_t gid = ((int64_t)blockIdx.x * kPoolThreads + threadIdx.x) / kTPG;
  const int sub = threadIdx.x % kTPG;
  const bool live = gid < 2 * p.groups_per_tensor;
  const int which = live && gid >= p.groups_per_tensor;
  const int64_t gg = live ? gid - which * p.groups_per_tensor : 0;  // (blk * B + b) * Hh + h
  const int h = (int)(gg % p.Hh);
  const int64_t rest = gg / p.Hh;
  const int b = (int)(rest % p.B);
  const int64_t blk = rest / p.B;
  const int64_t row_step = NAT ? (int64_t)p.Hh * (D / 8) : (D / 8);  // one token / one slot
  const uint4* base;
  if (NAT) {
    const int t = (int)(blk / ((int64_t)p.TH * p.TW));
    const int r = (int)(blk - (int64_t)t * p.TH * p.TW);
    const int i = r / p.TW, j = r - (r / p.TW) * p.TW;
    const int64_t N = (int64_t)p.T * p.H * p.W;
    base = (which ? k : q) +
           (((int64_t)b * N + ((int64_t)t * p.H + i * p.ph) * p.W + j * p.pw) * p.Hh + h) * (D / 8) +
           sub;
  } else {
    base = (which ? k : q) + (((int64_t)b * p.Hh + h) * p.Npad + blk * p.block) * (D / 8) + sub;
  }
  constexpr bool use_max = MAXP;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = use_max ? -INFINITY : 0.0;
  float mabs = 0.f;
  int cnt = 0;
  // rows [0, len) from `rowp`, in order, four loads ahead of the additions
  auto run = [&](const uint4* rowp, int len) {
    for (int c0 = 0; c0 < len; c0 += kAhead) {
      uint4 v[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (c0 + u < len) v[u] = __ldg(rowp + (int64_t)(c0 + u) * row_step);
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        if (c0 + u >= len) break;
        const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(pv[e]);
          if (use_max) {
            acc[2 * e] = fmax(acc[2 * e], (double)f.x);
            acc[2 * e + 1] = fmax(acc[2 * e + 1], (double)f.y);
          } else {
            acc[2 * e] = __dadd_rn(acc[2 * e], (double)f.x);
            acc[2 * e + 1] = __dadd_rn(acc[2 * e + 1], (double)f.y);
          }
          if (AMAX) mabs = fmaxf(mabs, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
    }
    cnt += len;
  };
  if (live) {
    if (NAT) {
      const int r = (int)(blk % ((int64_t)p.TH * p.TW));
      const int i = r / p.TW, j = r - (r / p.TW) * p.TW;
      const int hn = min(p.ph, p.H - i * p.ph), wn = min(p.pw, p.W - j * p.pw);
      for (int a = 0; a < hn; ++a) run(base + (int64_t)a * p.W * row_step, wn);
    } else {
      // runs of consecutive non-empty slots, 32 validity bits at a time
      const int64_t s0 = blk * p.block;
      for (int w0 = 0; w0 < p.block; w0 += 32) {
        const int64_t sl = s0 + w0;
        const int nb = min(32, p.block - w0);
        const int sh = (int)(sl & 31);
        uint32_t bits = __ldg(p.tile_valid + (sl >> 5)) >> sh;
        if (sh + nb > 32) bits |= __ldg(p.tile_valid + (sl >> 5) + 1) << (32 - sh);
        if (nb < 32) bits &= (1u << nb) - 1u;
        while (bits) {
          const int lo = __ffs(bits) - 1;
          const uint32_t rest_bits = ~(bits >> lo);
          const int len = rest_bits ? __ffs(rest_bits) - 1 : 32 - lo;
          run(base + (int64_t)(w0 + lo) * row_step, len);
          bits = (lo + len >= 32) ? 0u : bits & (~0u << (lo + len));
        }
      }
    }
    float* dst = p.ws + ((int64_t)which * p.groups_per_tensor +
                         ((int64_t)b * p.Hh + h) * p.nblocks + blk) * D + sub * 8;
    const double dc = (double)cnt;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      o[e] = __double2float_rn(cnt ? (use_max ? acc[e] : __ddiv_rn(acc[e], dc)) : 0.0);
    reinterpret_cast<float4*>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
  if (AMAX) {
    // max |x| of the group's tile: lanes of a group are kTPG consecutive lanes
#pragma unroll
    for (int o = kTPG / 2; o > 0; o >>= 1)
      mabs = fmaxf(mabs, __shfl_xor_sync(kFullMaskScore, mabs, o));
    if (live && sub == 0)
      atomicMax(p.amax + ((int64_t)which * p.B + b) * p.Hh + h, __float_as_uint(mabs));
  }
}

template <int D>
cudaError_t launch_pool(const Geometry& g, const uint32_t* tile_valid, const void* q, const void* k,
                        int use_max, bool natural, float* ws, uint32_t* amax, cudaStream_t st) {
  PoolParams p;
  p.B = g.B;
  p.Hh = g.Hh;
  p.T = g.T;
  p.H = g.H;
  p.W = g.W;
  p.ph = g.ph;
  p.pw = g.pw;
  p.TH = g.TH;
  p.TW = g.TW;
  p.block = g.block;
  p.nblocks = g.nblocks;
  p.Npad = g.Npad;
  p.groups_per_tensor = (int64_t)g.B * g.Hh * g.nblocks;
  p.use_max = use_max;
  p.tile_valid = tile_valid;
  p.amax = amax;
  p.ws = ws;
  const int64_t threads = 2 * p.groups_per_tensor * (D / 8);
  const unsigned grid = (unsigned)((threads + kPoolThreads - 1) / kPoolThreads);
  auto qq = reinterpret_cast<const uint4*>(q);
  auto kk = reinterpret_cast<const uint4*>(k);
  auto pick = [&](auto nat) {
    constexpr bool NAT = decltype(nat)::value;
    if (use_max)
      return amax ? draft_pool_kernel<D, NAT, true, true> : draft_pool_kernel<D, NAT, true, false>;
    return amax ? draft_pool_kernel<D, NAT, false, true> : draft_pool_kernel<D, NAT, false, false>;
  };
  auto kern = natural ? pick(std::true_type{}) : pick(std::false_type{});
  kern<<<grid, kPoolThreads, 0, st>>>(qq, kk, p);
  return cudaGetLastError();
}

// Unsigned key with the order of the floats (-0 and +0 equal; no NaN).
// Every non-NaN float maps above 0, so 0 can stand for "no candidate".
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(__fadd_rn(v, 0.0f));  // -0 + 0 = +0
  return (b >> 31) ? ~b : (b | 0x80000000u);
}
// The float of a key (inverse of order_key; -0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

// grid: (ceil(nblocks / R), Hh, B); R query rows per CTA.
template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    draft_score_topk_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                            int Hh, int nblocks, int R, int keep, int32_t* __restrict__ row_ptr,
                            int32_t* __restrict__ kv_idx, float* __restrict__ draft_map) {
  constexpr int kWarps = kScoreThreads / 32;
  constexpr int kKStride = D + 2;  // even: 8-byte loads of two channels, no bank conflicts
  extern __shared__ float2 shf2[];
  float* sq = reinterpret_cast<float*>(shf2);  // [kWarps][D][2]: rows w and w + kWarps
  float* sk = sq + 2 * kWarps * D;             // [kKeyChunk][kKStride]
  float* sl = sk + kKeyChunk * kKStride;       // [R][nblocks] logits
  uint8_t* sel = reinterpret_cast<uint8_t*>(sl + (int64_t)R * nblocks);  // [R][nblocks]
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * Hh + h;
  const int r0 = blockIdx.x * R;
  const int rows = min(R, nblocks - r0);  // R <= 2 * kWarps
  const float* qb = qbar + (bh * nblocks + r0) * D;
  const float* kb = kbar + bh * nblocks * D;
  // warp w carries rows w and w + kWarps: their values at channel c sit side
  // by side (one broadcast 8-byte load); missing rows read zeros
  for (int i = threadIdx.x; i < 2 * kWarps * D; i += kScoreThreads) {
    const int r = i / D, c = i - r * D;
    sq[((r % kWarps) * D + c) * 2 + r / kWarps] = r < rows ? qb[i] : 0.f;
  }
  for (int i = threadIdx.x; i < rows * nblocks; i += kScoreThreads) sel[i] = 0;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key chunks: the next chunk is loaded into registers while the current
  // one is used, then stored to shared memory (padded stride: no conflicts)
  constexpr int kPer = kKeyChunk * D / kScoreThreads;
  float pre[kPer];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * kScoreThreads;
      const int jj = idx / D, c = idx - jj * D;
      pre[u] = (j0 + jj < nblocks) ? kb[(int64_t)(j0 + jj) * D + c] : 0.f;
    }
  };
  load_chunk(0);
  for (int j0 = 0; j0 < nblocks; j0 += kKeyChunk) {
    const int nj = min(kKeyChunk, nblocks - j0);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * kScoreThreads;
      const int jj = idx / D, c = idx - jj * D;
      sk[jj * kKStride + c] = pre[u];
    }
    __syncthreads();
    if (j0 + kKeyChunk < nblocks) load_chunk(j0 + kKeyChunk);
    // warp w takes rows w and w + kWarps together (two independent chains);
    // lane = key block within the chunk.  Each logit is still the sequential
    // multiply-then-add over c.
    if (lane < nj && warp < rows) {
      const float2* kk = reinterpret_cast<const float2*>(sk + lane * kKStride);
      const float2* qq = reinterpret_cast<const float2*>(sq) + warp * D;
      float acc_a = 0.f, acc_b = 0.f;
#pragma unroll 4
      for (int c2 = 0; c2 < D / 2; ++c2) {
        const float2 kc = kk[c2];
        const float2 q0 = qq[2 * c2], q1 = qq[2 * c2 + 1];
        acc_a = __fadd_rn(acc_a, __fmul_rn(q0.x, kc.x));
        acc_b = __fadd_rn(acc_b, __fmul_rn(q0.y, kc.x));
        acc_a = __fadd_rn(acc_a, __fmul_rn(q1.x, kc.y));
        acc_b = __fadd_rn(acc_b, __fmul_rn(q1.y, kc.y));
      }
      sl[(int64_t)warp * nblocks + j0 + lane] = acc_a;
      if (warp + kWarps < rows) sl[(int64_t)(warp + kWarps) * nblocks + j0 + lane] = acc_b;
    }
  }
  __syncthreads();

  // top-k per row, one warp per row: k rounds of a warp-wide arg-max (larger
  // logit first, then the lower block index)
  for (int r = warp; r < rows; r += kWarps) {
    const float* L = sl + (int64_t)r * nblocks;
    uint8_t* sr = sel + (int64_t)r * nblocks;
    if (nblocks <= 32 * kRegCand) {
      // candidates j = lane + 32u held in registers as order-preserving
      // keys; `avail` marks the ones not yet taken.  A round takes the
      // largest key, then the lowest index among equal keys (two warp
      // reductions).
      uint32_t key[kRegCand];
      uint32_t avail = 0u;
#pragma unroll
      for (int u = 0; u < kRegCand; ++u) {
        const int j = lane + 32 * u;
        key[u] = j < nblocks ? order_key(L[j]) : 0u;
        if (j < nblocks) avail |= 1u << u;
      }
      const uint32_t start = avail;
      for (int it = 0; it < keep; ++it) {
        uint32_t bk = 0u;
        int bu = -1;
#pragma unroll
        for (int u = 0; u < kRegCand; ++u)
          if (((avail >> u) & 1u) && (bu < 0 || key[u] > bk)) {
            bk = key[u];
            bu = u;
          }
        const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t idx = (bu >= 0 && bk == top) ? (uint32_t)(lane + 32 * bu) : 0xffffffffu;
        const uint32_t win = __reduce_min_sync(0xffffffffu, idx);
        if (win != 0xffffffffu && (int)(win & 31u) == lane) avail &= ~(1u << (win >> 5));
      }
#pragma unroll
      for (int u = 0; u < kRegCand; ++u) {
        const int j = lane + 32 * u;
        if (j < nblocks) sr[j] = (((start & ~avail) >> u) & 1u) ? 1 : 0;
      }
      __syncwarp();
    } else {
      for (int it = 0; it < keep; ++it) {
        float best = -FLT_MAX;
        int bidx = 0x7fffffff;
        for (int j = lane; j < nblocks; j += 32) {
          if (sr[j]) continue;
          const float v = L[j];
          if (bidx == 0x7fffffff || v > best || (v == best && j < bidx)) {
            best = v;
            bidx = j;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, best, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
          const bool take = (oi != 0x7fffffff) &&
                            (bidx == 0x7fffffff || ov > best || (ov == best && oi < bidx));
          if (take) {
            best = ov;
            bidx = oi;
          }
        }
        if (lane == 0 && bidx != 0x7fffffff) sr[bidx] = 1;
        __syncwarp();
      }
    }
    // ascending output
    const int64_t grow = bh * nblocks + r0 + r;
    int32_t* out = kv_idx + grow * keep;
    int pos = 0;
    for (int j0 = 0; j0 < nblocks; j0 += 32) {
      const int j = j0 + lane;
      const bool on = j < nblocks && sr[j];
      const uint32_t bal = __ballot_sync(0xffffffffu, on);
      if (on) {
        const int at = pos + __popc(bal & ((1u << lane) - 1u));
        if (at < keep) out[at] = j;
      }
      pos += __popc(bal);
    }
    if (row_ptr && lane == 0) {
      row_ptr[grow] = (int32_t)(grow * keep);
      if (grow == (int64_t)gridDim.z * Hh * nblocks - 1) row_ptr[grow + 1] = (int32_t)((grow + 1) * keep);
    }
    if (draft_map) {
      double mx = -DBL_MAX;
      for (int j = lane; j < nblocks; j += 32) mx = fmax(mx, (double)L[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const double inv_sqrt_d = 1.0 / sqrt((double)D);
      double sum = 0.0;
      for (int j = lane; j < nblocks; j += 32) sum += exp(((double)L[j] - mx) * inv_sqrt_d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      float* dm = draft_map + grow * nblocks;
      for (int j = lane; j < nblocks; j += 32)
        dm[j] = (float)(exp(((double)L[j] - mx) * inv_sqrt_d) / sum);
    }
  }
}

// ---------------------------------------------------------------------------
// Scoring with the logits in registers (up to 512 key blocks per row).
//
// A warp owns R whole query-block rows; lane l accumulates the logits of key
// blocks j = l + 32u (u < U) of each row, so a row's top-k runs straight out
// of registers and no logit ever goes to shared memory.  Rows are held in
// pairs, one fp32 pair per key, and updated with the two-wide fp32 multiply
// and add (each lane of the pair rounded on its own, so every logit is still
// the sequential multiply-then-add chain over c = 0..D-1).  The CTA's warps
// share the pooled keys, staged CK channels at a time in a two-stage
// cp.async ring as [channel quad][key][4] (a lane reads four channels of one
// key with one 16-byte load; a warp's loads are contiguous); the pooled query
// values are staged as [channel][row], so a row pair is one broadcast load.
// ---------------------------------------------------------------------------
constexpr int kRegScoreWarps = 4;
constexpr int kRegScoreCK = 16;  // channels per stage

__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int U>
struct RegScoreCfg {
  static constexpr int R = 4;                          // rows per warp (pairs)
  static constexpr int kRows = R * kRegScoreWarps;     // rows per CTA
  static constexpr int NK = 32 * U;                    // keys, padded
  static constexpr int kStageK = kRegScoreCK * NK;     // floats per K stage
  static constexpr int kStageQ = kRegScoreCK * kRows;  // floats per Q stage
  static constexpr size_t kSmem = 2 * (size_t)(kStageK + kStageQ) * sizeof(float);
};

// grid: (ceil(nblocks / kRows), Hh, B)
template <int D, int U>
__global__ void __launch_bounds__(32 * kRegScoreWarps, U <= 12 ? 4 : 3)
    draft_score_reg_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                           int Hh, int nblocks, int keep, int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ kv_idx, float* __restrict__ draft_map) {
  using Cfg = RegScoreCfg<U>;
  constexpr int R = Cfg::R, RP = R / 2, CK = kRegScoreCK, NK = Cfg::NK;
  constexpr int kThreads = 32 * kRegScoreWarps;
  static_assert(D % CK == 0 && CK % 4 == 0 && R % 2 == 0, "staging shape");
  extern __shared__ float4 shf4[];
  float* sK = reinterpret_cast<float*>(shf4);  // [2][CK/4][NK][4]
  float* sQ = sK + 2 * Cfg::kStageK;            // [2][CK][kRows]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * Hh + h;
  const int r0 = blockIdx.x * Cfg::kRows;
  const float* qb = qbar + bh * nblocks * D;
  const float* kb = kbar + bh * nblocks * D;

  // stage `st` <- channels [c0, c0 + CK); entries past the grid are
  // zero-filled (a valid source address is still passed: the copy reads 0
  // bytes from it)
  auto issue = [&](int st, int c0) {
    float* dk = sK + st * Cfg::kStageK;
    for (int i = threadIdx.x; i < Cfg::kStageK / 4; i += kThreads) {
      const int c4 = i / NK, j = i - c4 * NK;
      const bool ok = j < nblocks;
      cp_async16(dk + 4 * i, kb + (int64_t)(ok ? j : 0) * D + c0 + 4 * c4, ok);
    }
    float* dq = sQ + st * Cfg::kStageQ;
    for (int i = threadIdx.x; i < Cfg::kStageQ; i += kThreads) {
      const int r = i / CK, c = i - r * CK;
      const bool ok = r0 + r < nblocks;
      cp_async4(dq + c * Cfg::kRows + r, qb + (int64_t)(ok ? r0 + r : 0) * D + c0 + c, ok);
    }
    cp_async_commit();
  };

  uint64_t acc[RP][U];  // (row 2p, row 2p + 1) of key lane + 32u
#pragma unroll
  for (int rp = 0; rp < RP; ++rp)
#pragma unroll
    for (int u = 0; u < U; ++u) acc[rp][u] = f2(0.f, 0.f);

  issue(0, 0);
  constexpr int kStages = D / CK;
  for (int cs = 0; cs < kStages; ++cs) {
    if (cs + 1 < kStages) {
      issue((cs + 1) & 1, (cs + 1) * CK);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float4* ck = reinterpret_cast<const float4*>(sK + (cs & 1) * Cfg::kStageK) + lane;
    const float* cq = sQ + (cs & 1) * Cfg::kStageQ + warp * R;
#pragma unroll
    for (int c4 = 0; c4 < CK / 4; ++c4) {
      uint64_t qp[4][RP];  // channel 4*c4 + e of rows (2p, 2p + 1)
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int rp = 0; rp < RP; ++rp)
          qp[e][rp] = *reinterpret_cast<const uint64_t*>(cq + (4 * c4 + e) * Cfg::kRows + 2 * rp);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float4 kv = ck[c4 * NK + 32 * u];  // channels 4*c4 .. 4*c4 + 3 of key lane + 32u
        const float ke[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t kk = f2(ke[e], ke[e]);
#pragma unroll
          for (int rp = 0; rp < RP; ++rp) acc[rp][u] = fadd2(acc[rp][u], fmul2(qp[e][rp], kk));
        }
      }
    }
    __syncthreads();  // the next issue() overwrites this stage
  }

  // top-k of each row (larger logit first, then the lower block index).
  // The k-th largest key T is found bit by bit from the top (the largest T
  // with at least k keys >= T), for the warp's R rows side by side; then
  // every key above T is taken, and of the keys equal to T the ones with the
  // lowest block indices.  Blocks past the grid (and rows past it) hold key
  // 0, below every real key.
  uint32_t key[R][U];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const bool row_in = r0 + warp * R + r < nblocks;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float lo, hi;
      unf2(acc[r >> 1][u], lo, hi);
      key[r][u] = (row_in && lane + 32 * u < nblocks) ? order_key((r & 1) ? hi : lo) : 0u;
    }
  }
  uint32_t T[R];
#pragma unroll
  for (int r = 0; r < R; ++r) T[r] = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    unsigned tot[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t cand = T[r] | (1u << bit);
      unsigned c = 0;
#pragma unroll
      for (int u = 0; u < U; ++u) c += key[r][u] >= cand ? 1u : 0u;
      tot[r] = __reduce_add_sync(kFullMaskScore, c);
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (tot[r] >= (unsigned)keep) T[r] |= 1u << bit;
  }
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = r0 + warp * R + r;
    if (row >= nblocks) break;  // warp-uniform
    unsigned c_gt = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) c_gt += key[r][u] > T[r] ? 1u : 0u;
    int eq_left = keep - (int)__reduce_add_sync(kFullMaskScore, c_gt);
    uint32_t taken = 0u;
#pragma unroll
    for (int u = 0; u < U; ++u) {  // block order: u, then lane
      const bool eq = key[r][u] == T[r];
      const uint32_t bal = __ballot_sync(kFullMaskScore, eq);
      if (key[r][u] > T[r] || (eq && __popc(bal & below) < eq_left)) taken |= 1u << u;
      eq_left -= __popc(bal);
    }
    // ascending output: j = 32u + lane grows with (u, lane)
    const int64_t grow = bh * nblocks + row;
    int32_t* out = kv_idx + grow * keep;
    int pos = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool on = (taken >> u) & 1u;
      const uint32_t bal = __ballot_sync(kFullMaskScore, on);
      if (on) {
        const int at = pos + __popc(bal & below);
        if (at < keep) out[at] = lane + 32 * u;
      }
      pos += __popc(bal);
    }
    if (row_ptr && lane == 0) {
      row_ptr[grow] = (int32_t)(grow * keep);
      if (grow == (int64_t)gridDim.z * Hh * nblocks - 1) row_ptr[grow + 1] = (int32_t)((grow + 1) * keep);
    }
    if (draft_map) {
      double lv[U];  // the logits back from their keys (the map is exact to them)
#pragma unroll
      for (int u = 0; u < U; ++u) lv[u] = (double)key_value(key[r][u]);
      double mx = -DBL_MAX;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks) mx = fmax(mx, lv[u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFullMaskScore, mx, o));
      const double inv_sqrt_d = 1.0 / sqrt((double)D);
      double sum = 0.0;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks) sum += exp((lv[u] - mx) * inv_sqrt_d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFullMaskScore, sum, o);
      float* dm = draft_map + grow * nblocks;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks) dm[lane + 32 * u] = (float)(exp((lv[u] - mx) * inv_sqrt_d) / sum);
    }
  }
}

template <int D, int U>
cudaError_t launch_score_reg(const Geometry& g, const float* ws, int keep, int32_t* row_ptr,
                             int32_t* kv_idx, float* draft_map, cudaStream_t st) {
  using Cfg = RegScoreCfg<U>;
  auto kern = draft_score_reg_kernel<D, U>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Cfg::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t groups = (int64_t)g.B * g.Hh * g.nblocks;
  const dim3 grid((unsigned)((g.nblocks + Cfg::kRows - 1) / Cfg::kRows), (unsigned)g.Hh,
                  (unsigned)g.B);
  kern<<<grid, 32 * kRegScoreWarps, Cfg::kSmem, st>>>(ws, ws + groups * D, g.Hh, (int)g.nblocks,
                                                       keep, row_ptr, kv_idx, draft_map);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_t(const Geometry& g, const uint32_t* tile_valid, const void* q, const void* k,
                     int keep, int pooling, bool natural, int32_t* row_ptr, int32_t* kv_idx,
                     float* draft_map, float* ws, unsigned int* status, uint64_t wait_limit_ns,
                     cudaStream_t st, uint32_t* amax, bool* amax_recorded) {
  const int use_max = pooling == BSA_POOL_MAX ? 1 : 0;
  cudaError_t e = launch_pool<D>(g, tile_valid, q, k, use_max, natural, ws, amax, st);
  if (e != cudaSuccess) return e;
  if (amax_recorded) *amax_recorded = amax != nullptr;
  // rows of up to 512 key blocks: logits in registers
  // (one kernel per 32-block width U: no padded keys beyond the next 32)
  if (g.nblocks <= 512) {
    switch ((g.nblocks + 31) / 32) {
#define BSA_SCORE_U(u) \
  case u:              \
    return launch_score_reg<D, u>(g, ws, keep, row_ptr, kv_idx, draft_map, st);
      BSA_SCORE_U(1) BSA_SCORE_U(2) BSA_SCORE_U(3) BSA_SCORE_U(4) BSA_SCORE_U(5) BSA_SCORE_U(6)
      BSA_SCORE_U(7) BSA_SCORE_U(8) BSA_SCORE_U(9) BSA_SCORE_U(10) BSA_SCORE_U(11)
      BSA_SCORE_U(12) BSA_SCORE_U(13) BSA_SCORE_U(14) BSA_SCORE_U(15) BSA_SCORE_U(16)
#undef BSA_SCORE_U
      default:
        break;
    }
  }
  const int R = draft_rows_per_cta(g.nblocks);
  const size_t smem = (size_t)(2 * (kScoreThreads / 32) * D + kKeyChunk * (D + 2) +
                               (int64_t)R * g.nblocks) * sizeof(float) +
                      (size_t)R * g.nblocks;
  auto kern = draft_score_topk_kernel<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((g.nblocks + R - 1) / R), (unsigned)g.Hh, (unsigned)g.B);
  const int64_t groups = (int64_t)g.B * g.Hh * g.nblocks;
  kern<<<grid, kScoreThreads, smem, st>>>(ws, ws + groups * D, g.Hh, (int)g.nblocks, R, keep,
                                          row_ptr, kv_idx, draft_map);
  return cudaGetLastError();
}

}  // namespace

int draft_rows_per_cta(int64_t nblocks) {
  // logits + selection flags of R rows within ~150 KB of shared memory; at
  // most two rows per warp of the scoring kernel
  static_assert(2 * (kScoreThreads / 32) >= 16, "two rows per warp");
  int64_t R = 16;
  while (R > 1 && R * nblocks * 5 > 150 * 1024) R >>= 1;
  return (int)R;
}

size_t draft_workspace_bytes(const Geometry& g) {
  return (size_t)2 * g.B * g.Hh * g.nblocks * g.D * sizeof(float);
}

cudaError_t launch_draft_mask(const Geometry& g, const uint32_t* tile_valid, const void* q,
                              const void* k, int keep, int pooling, int32_t* row_ptr,
                              int32_t* kv_idx, float* draft_map, float* ws, unsigned int* status,
                              uint64_t wait_limit_ns, cudaStream_t st, bool natural,
                              uint32_t* amax, bool* amax_recorded) {
  if (g.D == 128)
    return launch_t<128>(g, tile_valid, q, k, keep, pooling, natural, row_ptr, kv_idx, draft_map,
                         ws, status, wait_limit_ns, st, amax, amax_recorded);
  return launch_t<64>(g, tile_valid, q, k, keep, pooling, natural, row_ptr, kv_idx, draft_map, ws,
                      status, wait_limit_ns, st, amax, amax_recorded);
}

}  // namespace bsa

// ---------------------------------------------------------------------------
// Draft mask without any allocation by the caller.
//
// Some callers cannot allocate device memory of their own: for example a
// plugin running inside a host program that owns every device allocation and
// hands the plugin only its input and output buffers, or a caller held to a
// fixed memory budget, where an extra allocation may fail or stall the device
// in the middle of a step.  bsa_draft_mask_noalloc serves them: it computes
// exactly what bsa_draft_mask computes, with its fp64 scratch (the pooled Q
// and K) taken from the file-scope device array below instead of a caller
// workspace.
//
// The array is kNoAllocScratchBytes (32 MiB) on every GPU that loads this
// library, held until the process exits; problems whose scratch would exceed
// it (2*B*Hh*Nb*D*8 bytes) are rejected.  Every call on a device shares the
// one array, so calls whose kernels overlap on the GPU (on different streams,
// or from different host threads) race on it; calls in order on one stream
// are safe.  The array keeps the last call's contents: nothing needs clearing,
// because the pooling kernel writes every element the scoring kernel reads.
// ---------------------------------------------------------------------------
#include <mutex>

namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_noalloc_scratch on the current device.  Looked up once
// per device, on the first call made with that device current, and cached
// for the life of the process: after cudaDeviceReset the cached address no
// longer names live memory, so the entry point must not be called again in
// that process.
cudaError_t noalloc_scratch_address(float** out) {
  static std::mutex mu;
  static float* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = reinterpret_cast<float*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_draft_noalloc_max_scratch_bytes(void) { return bsa::kNoAllocScratchBytes; }

extern "C" bsa_status bsa_draft_mask_noalloc(bsa_plan_t plan, const void* q_slots,
                                             const void* k_slots, int sparsity_pct,
                                             int32_t* row_ptr, int32_t* kv_idx, float* draft_map,
                                             void* stream) {
  using namespace bsa;
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_TILE) return set_error(BSA_ERR_INVALID_ARG, "draft mask needs a TILE plan");
  if (sparsity_pct < 0 || sparsity_pct >= 100)
    return set_error(BSA_ERR_INVALID_ARG, "sparsity must be in [0, 100)");
  if (!q_slots || !k_slots || !kv_idx)
    return set_error(BSA_ERR_INVALID_ARG, "q_slots / k_slots / kv_idx is NULL");
  if (!aligned16(q_slots) || !aligned16(k_slots))
    return set_error(BSA_ERR_ALIGNMENT, "q_slots / k_slots not 16-byte aligned");
  const size_t need = draft_workspace_bytes(g);
  if (need > kNoAllocScratchBytes)
    return set_error(BSA_ERR_UNSUPPORTED,
                     "draft scratch of " + std::to_string(need) +
                         " bytes exceeds the 32 MiB static scratch of bsa_draft_mask_noalloc; "
                         "use bsa_draft_mask with a caller workspace");
  if (g.nblocks > 18000) return set_error(BSA_ERR_UNSUPPORTED, "draft mask supports up to 18000 blocks");
  if ((int64_t)g.B * g.Hh * g.Npad >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "draft mask needs B*Hh*Npad < 2^31");
  const int keep = (int)((g.nblocks * (100 - sparsity_pct) + 99) / 100);
  if ((int64_t)g.B * g.Hh * g.nblocks * keep >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev != plan->device)
    return set_error(BSA_ERR_INVALID_ARG,
                     "the current device is not the plan's: the static scratch of one device "
                     "cannot serve a plan of another");
  float* scratch = nullptr;
  e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(scratch)");
  e = launch_draft_mask(g, plan->d_tile_valid, q_slots, k_slots, keep, plan->draft_pooling, row_ptr,
                        kv_idx, draft_map, scratch, plan->d_status, plan->wait_limit_ns,
                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask_noalloc launch");
}
