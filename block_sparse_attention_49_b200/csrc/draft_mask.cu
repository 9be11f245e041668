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
//         and is divided once by the token count.  With max pooling (which
//         the article's authors tried before settling on the average) it is
//         the channel-wise maximum instead, exact in any order.  Written as
//         fp32 (rounded once), and in the default fp64 precision also as
//         fp64 with an upper bound of each vector's 2-norm.  16-byte loads,
//         four rows ahead; HBM bound.
//  score: for a group of query-block rows of one (b, head), the logits
//         L[i][j] = sum_c qbar_i[c]*kbar_j[c], sequential over c, the
//         product and the sum each rounded (no fused multiply-add), in the
//         plan's precision; per row the k largest, ties to the lower j,
//         written ascending.  Optionally the draft map
//         softmax_j(L[i][j]/sqrt(D)), evaluated in fp64 and stored as fp32.
//         The fp64 lists come out of fp32 logits and a proven bound on their
//         distance to the fp64 ones (see draft_score_reg_kernel).
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
constexpr unsigned kFullMaskScore = 0xffffffffu;

// ---------------------------------------------------------------------------
// Pooling.  One group of D/8 threads per unit (Q or K, tile, batch, head);
// each thread owns 8 channels: eight independent fp64 chains, each the
// sequential sum over the tile's tokens in row-major order, stored as fp32.  Token rows are
// read with 16-byte streaming loads (no L1 allocation), four rows ahead of the additions.  Units are
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
  // pooled Q then K: fp32 always; with F64 first the fp64 values, then the
  // fp32 copies, then the fp32 2-norms (rounded up) of the fp64 values
  void* ws;
};

template <int D, bool NAT, bool MAXP, bool AMAX, bool F64>
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
  double ss = 0.0;  // F64: this thread's share of the squared 2-norm
  int cnt = 0;
  // rows [0, len) from `rowp`, in order, four loads ahead of the additions
  auto run = [&](const uint4* rowp, int len) {
    for (int c0 = 0; c0 < len; c0 += kAhead) {
      uint4 v[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (c0 + u < len) v[u] = ld_stream_v4(rowp + (int64_t)(c0 + u) * row_step);
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
    const int64_t at = ((int64_t)which * p.groups_per_tensor +
                        ((int64_t)b * p.Hh + h) * p.nblocks + blk) * D + sub * 8;
    const double dc = (double)cnt;
    double o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = cnt ? (use_max ? acc[e] : __ddiv_rn(acc[e], dc)) : 0.0;
    const int64_t n_all = 2 * p.groups_per_tensor * D;  // values of Q and K
    float* ws32 = static_cast<float*>(p.ws);
    if (F64) {
      double2* dst = reinterpret_cast<double2*>(static_cast<double*>(p.ws) + at);
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = make_double2(o[2 * e], o[2 * e + 1]);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fma(o[e], o[e], ss);
      ws32 = reinterpret_cast<float*>(static_cast<double*>(p.ws) + n_all);
    }
    float4* dst = reinterpret_cast<float4*>(ws32 + at);
    dst[0] = make_float4(__double2float_rn(o[0]), __double2float_rn(o[1]),
                         __double2float_rn(o[2]), __double2float_rn(o[3]));
    dst[1] = make_float4(__double2float_rn(o[4]), __double2float_rn(o[5]),
                         __double2float_rn(o[6]), __double2float_rn(o[7]));
  }
  if (F64) {
    // 2-norm of the unit's fp64 values, an upper bound: the squares' sum in
    // fp64 (relative error below D * 2^-53), its square root grown by 2^-40
    // and rounded up to fp32.  Lanes of a group are kTPG consecutive lanes.
#pragma unroll
    for (int o = kTPG / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(kFullMaskScore, ss, o);
    if (live && sub == 0) {
      float* norms = reinterpret_cast<float*>(static_cast<double*>(p.ws) +
                                              2 * p.groups_per_tensor * D) +
                     2 * p.groups_per_tensor * D;
      norms[(int64_t)which * p.groups_per_tensor + ((int64_t)b * p.Hh + h) * p.nblocks + blk] =
          __double2float_ru(sqrt(ss) * (1.0 + 0x1p-40));
    }
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
                        int use_max, bool natural, bool f64, void* ws, uint32_t* amax,
                        cudaStream_t st) {
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
  auto pick = [&](auto nat, auto wide) {
    constexpr bool NAT = decltype(nat)::value, F64 = decltype(wide)::value;
    if (use_max)
      return amax ? draft_pool_kernel<D, NAT, true, true, F64>
                  : draft_pool_kernel<D, NAT, true, false, F64>;
    return amax ? draft_pool_kernel<D, NAT, false, true, F64>
                : draft_pool_kernel<D, NAT, false, false, F64>;
  };
  auto kern = natural ? (f64 ? pick(std::true_type{}, std::true_type{})
                             : pick(std::true_type{}, std::false_type{}))
                      : (f64 ? pick(std::false_type{}, std::true_type{})
                             : pick(std::false_type{}, std::false_type{}));
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

__device__ __forceinline__ float mul_rn(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ double mul_rn(double a, double b) { return __dmul_rn(a, b); }
__device__ __forceinline__ float add_rn(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ double add_rn(double a, double b) { return __dadd_rn(a, b); }

// grid: (ceil(nblocks / R), Hh, B); R query rows per CTA.  Rows of more than
// 512 key blocks: the logits of R rows in shared memory.
template <int D, typename T>
__global__ void __launch_bounds__(kScoreThreads)
    draft_score_topk_kernel(const T* __restrict__ qbar, const T* __restrict__ kbar, int Hh,
                            int nblocks, int R, int keep, int32_t* __restrict__ row_ptr,
                            int32_t* __restrict__ kv_idx, float* __restrict__ draft_map) {
  using T2 = typename std::conditional<std::is_same<T, double>::value, double2, float2>::type;
  constexpr int kWarps = kScoreThreads / 32;
  constexpr int kKStride = D + 2;  // even: two-channel loads, no bank conflicts
  extern __shared__ double4 shd4[];
  T* sq = reinterpret_cast<T*>(shd4);      // [kWarps][D][2]: rows w and w + kWarps
  T* sk = sq + 2 * kWarps * D;             // [kKeyChunk][kKStride]
  T* sl = sk + kKeyChunk * kKStride;       // [R][nblocks] logits
  uint8_t* sel = reinterpret_cast<uint8_t*>(sl + (int64_t)R * nblocks);  // [R][nblocks]
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * Hh + h;
  const int r0 = blockIdx.x * R;
  const int rows = min(R, nblocks - r0);  // R <= 2 * kWarps
  const T* qb = qbar + (bh * nblocks + r0) * D;
  const T* kb = kbar + bh * nblocks * D;
  // warp w carries rows w and w + kWarps: their values at channel c sit side
  // by side (one broadcast load); missing rows read zeros
  for (int i = threadIdx.x; i < 2 * kWarps * D; i += kScoreThreads) {
    const int r = i / D, c = i - r * D;
    sq[((r % kWarps) * D + c) * 2 + r / kWarps] = r < rows ? qb[i] : T(0);
  }
  for (int i = threadIdx.x; i < rows * nblocks; i += kScoreThreads) sel[i] = 0;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key chunks: the next chunk is loaded into registers while the current
  // one is used, then stored to shared memory (padded stride: no conflicts)
  constexpr int kPer = kKeyChunk * D / kScoreThreads;
  T pre[kPer];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * kScoreThreads;
      const int jj = idx / D, c = idx - jj * D;
      pre[u] = (j0 + jj < nblocks) ? kb[(int64_t)(j0 + jj) * D + c] : T(0);
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
      const T2* kk = reinterpret_cast<const T2*>(sk + lane * kKStride);
      const T2* qq = reinterpret_cast<const T2*>(sq) + warp * D;
      T acc_a = T(0), acc_b = T(0);
#pragma unroll 4
      for (int c2 = 0; c2 < D / 2; ++c2) {
        const T2 kc = kk[c2];
        const T2 q0 = qq[2 * c2], q1 = qq[2 * c2 + 1];
        acc_a = add_rn(acc_a, mul_rn(q0.x, kc.x));
        acc_b = add_rn(acc_b, mul_rn(q0.y, kc.x));
        acc_a = add_rn(acc_a, mul_rn(q1.x, kc.y));
        acc_b = add_rn(acc_b, mul_rn(q1.y, kc.y));
      }
      sl[(int64_t)warp * nblocks + j0 + lane] = acc_a;
      if (warp + kWarps < rows) sl[(int64_t)(warp + kWarps) * nblocks + j0 + lane] = acc_b;
    }
  }
  __syncthreads();

  // top-k per row, one warp per row: k rounds of a warp-wide arg-max (larger
  // logit first, then the lower block index)
  for (int r = warp; r < rows; r += kWarps) {
    const T* L = sl + (int64_t)r * nblocks;
    uint8_t* sr = sel + (int64_t)r * nblocks;
    for (int it = 0; it < keep; ++it) {
      T best = T(0);
      int bidx = 0x7fffffff;
      for (int j = lane; j < nblocks; j += 32) {
        if (sr[j]) continue;
        const T v = L[j];
        if (bidx == 0x7fffffff || v > best) {  // j ascends: equal values keep the lower j
          best = v;
          bidx = j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const T ov = __shfl_xor_sync(0xffffffffu, best, o);
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
// A warp owns R whole query-block rows; lane l accumulates the fp32 logits
// of key blocks j = l + 32u (u < U) of each row, so a row's top-k runs
// straight out of registers and no logit ever goes to shared memory.  Every
// logit is the sequential multiply-then-add chain over c = 0..D-1, each
// operation rounded to fp32.  Rows are held in pairs, one fp32 pair per key,
// updated with the two-wide fp32 multiply and add (each lane of the pair
// rounded on its own).  Keys are staged 16 channels at a time as [channel
// quad][key][4], so a lane reads four channels of one key with one 16-byte
// load and a warp's loads are contiguous; the pooled query values are
// staged as [channel][row] and read by broadcast.  For the default fp64
// lists the fp32 logits decide every block that lies clearly above or below
// the k-th, and the rest get their fp64 logits (CERT).
// ---------------------------------------------------------------------------
constexpr int kRegScoreWarps = 4;

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
  static constexpr int CK = 16;                        // channels per stage
  static constexpr int kRows = R * kRegScoreWarps;     // rows per CTA
  static constexpr int NK = 32 * U;                    // keys, padded
  static constexpr int kStageK = CK * NK;              // floats per K stage
  static constexpr int kStageQ = CK * kRows;           // floats per Q stage
  static constexpr size_t kSmem = 2 * (size_t)(kStageK + kStageQ) * sizeof(float);
  // the fp64 refinement's per-warp list of (logit, block) in the same space
  static_assert(kRegScoreWarps * NK * 12 <= (int)kSmem, "refinement list fits");
};

// |fp32 logit - fp64 logit| <= kErrBound * |qbar| * |kbar| + 2^-100 for the
// sequential unfused chains of D products: gamma_D(fp32) on the fp32 chain
// (of inputs within 2^-24 of the fp64 ones: (1 + 2^-24)^2 - 1 on each
// product) plus gamma_D(fp64) on the fp64 chain, where gamma_n = n u / (1 -
// n u) (Higham, "Accuracy and Stability of Numerical Algorithms", sections
// 3.1 and 3.5), and sum |q_c k_c| <= |q| |k|; doubled as a margin.  The
// absolute term covers fp32 underflow.
template <int D>
struct ErrBound {
  static constexpr double u32 = 0x1p-24, u64 = 0x1p-53;
  static constexpr double g32 = D * u32 / (1.0 - D * u32), g64 = D * u64 / (1.0 - D * u64);
  static constexpr double value = 2.0 * (g32 * (1.0 + u32) * (1.0 + u32) + 2.0 * u32 + u32 * u32 + g64);
};

// The fp64 logit of query block `qr` and key block `kr` (D values each),
// computed by the whole warp: lanes form the rounded products, then every
// lane adds them in channel order.
template <int D>
__device__ __forceinline__ double warp_logit64(const double* qr, const double* kr, int lane) {
  double pr[D / 32];
#pragma unroll
  for (int m = 0; m < D / 32; ++m) pr[m] = __dmul_rn(qr[lane + 32 * m], kr[lane + 32 * m]);
  double L = 0.0;
#pragma unroll
  for (int c = 0; c < D; ++c) L = __dadd_rn(L, __shfl_sync(kFullMaskScore, pr[c >> 5], c & 31));
  return L;
}

// Ranks a row's band (bit u of `band`: key block lane + 32u) on the fp64
// logits and adds the `need` largest (then lowest block index) to `taken`.
// sv / sj: this warp's list space in shared memory (NK entries).  Kept out
// of line: it runs for few rows, and its registers stay out of the scorer's.
template <int D, int U>
__device__ __noinline__ uint32_t rank_band64(const double* __restrict__ qr,
                                            const double* __restrict__ khead, uint32_t band,
                                            int need, uint32_t taken, int lane, double* sv,
                                            int* sj) {
  int cnt = 0;
#pragma unroll 1
  for (int u = 0; u < U; ++u) {
    uint32_t bb = __ballot_sync(kFullMaskScore, (band >> u) & 1u);
    while (bb) {
      const int j = (__ffs(bb) - 1) + 32 * u;
      bb &= bb - 1;
      const double L = warp_logit64<D>(qr, khead + (int64_t)j * D, lane);
      if (lane == 0) {
        sv[cnt] = L;
        sj[cnt] = j;
      }
      ++cnt;
    }
  }
  __syncwarp();
  for (int it = 0; it < need; ++it) {
    double best = 0.0;
    int bj = 0x7fffffff, be = -1;
    for (int x = lane; x < cnt; x += 32) {
      const int j = sj[x];
      if (j < 0) continue;
      const double v = sv[x];
      if (be < 0 || v > best || (v == best && j < bj)) {
        best = v;
        bj = j;
        be = x;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(kFullMaskScore, best, o);
      const int oj = __shfl_xor_sync(kFullMaskScore, bj, o);
      const int oe = __shfl_xor_sync(kFullMaskScore, be, o);
      if (oe >= 0 && (be < 0 || ov > best || (ov == best && oj < bj))) {
        best = ov;
        bj = oj;
        be = oe;
      }
    }
    if (be >= 0) {
      if (lane == (bj & 31)) taken |= 1u << (bj >> 5);
      if (lane == 0) sj[be] = -1;
    }
    __syncwarp();
  }
  return taken;
}

// The fp64 logits of one row for the draft map (lane's keys lane + 32u).
template <int D, int U>
__device__ __noinline__ void row_logits64(const double* __restrict__ qr,
                                          const double* __restrict__ khead, int nblocks, int lane,
                                          double* lv) {
#pragma unroll 1
  for (int u = 0; u < U; ++u) {
    double a = 0.0;
    if (lane + 32 * u < nblocks) {
      const double* kr = khead + (int64_t)(lane + 32 * u) * D;
      for (int c = 0; c < D; ++c) a = __dadd_rn(a, __dmul_rn(qr[c], kr[c]));
    }
    lv[u] = a;
  }
}

// grid: (ceil(nblocks / kRows), Hh, B).  CERT: the plan's precision is fp64;
// the fp32 logits pick the blocks that are certain under the error bound,
// and only the ones within it of the k-th logit get their fp64 logits (from
// q64 / k64), so the lists are those of the fp64 chains.
template <int D, int U, bool CERT>
__global__ void __launch_bounds__(32 * kRegScoreWarps, U <= 12 ? 4 : 3)
    draft_score_reg_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                           int Hh, int nblocks, int keep, int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ kv_idx, float* __restrict__ draft_map,
                           const double* __restrict__ q64, const double* __restrict__ k64,
                           const float* __restrict__ qnorm, const float* __restrict__ knorm) {
  using Cfg = RegScoreCfg<U>;
  constexpr int R = Cfg::R, RP = R / 2, CK = Cfg::CK, NK = Cfg::NK;
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
    __syncthreads();  // the next issue() overwrites this stage (or the refinement lists)
  }

  // top-k of each row (larger logit first, then the lower block index).
  // The k-th largest key T is found bit by bit from the top (the largest T
  // with at least k keys >= T), for the warp's R rows side by side; then
  // every key above T is taken, and of the keys equal to T the ones with the
  // lowest block indices.  Blocks past the grid (and rows past it) hold key
  // 0, below every real key.  With fp32 lists the search stops once every
  // row has exactly k keys >= its prefix Tk: those k keys are the selection
  // whatever the remaining bits, and the tie rule on Tk takes all of them.
  // (The fp64 lists' kernel runs every bit: stopping early measured slower
  // there, although the result is the same.)
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
  uint32_t Tk[R];
  unsigned nge[R];  // keys >= Tk[r]; rows past the grid count as settled
#pragma unroll
  for (int r = 0; r < R; ++r) {
    Tk[r] = 0u;
    nge[r] = r0 + warp * R + r < nblocks ? 32u * U : (unsigned)keep;
  }
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    if constexpr (!CERT) {
      bool settled = true;
#pragma unroll
      for (int r = 0; r < R; ++r) settled = settled && nge[r] == (unsigned)keep;
      if (settled) break;  // warp-uniform: the counts are warp sums
    }
    unsigned tot[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t cand = Tk[r] | (1u << bit);
      unsigned c = 0;
#pragma unroll
      for (int u = 0; u < U; ++u) c += key[r][u] >= cand ? 1u : 0u;
      tot[r] = __reduce_add_sync(kFullMaskScore, c);
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (tot[r] >= (unsigned)keep) {
        Tk[r] |= 1u << bit;
        nge[r] = tot[r];
      }
  }
  float kmax = 0.f;  // CERT: the largest key-block norm of this (b, head)
  if constexpr (CERT) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (lane + 32 * u < nblocks) kmax = fmaxf(kmax, knorm[bh * nblocks + lane + 32 * u]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(kFullMaskScore, kmax, o));
  }
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = r0 + warp * R + r;
    if (row >= nblocks) break;  // warp-uniform
    uint32_t taken = 0u;
    bool by_index = true;
    if constexpr (CERT) {
      // blocks whose fp32 logit lies more than twice the bound above the
      // k-th one are in, more than twice below it out, whatever the fp64
      // logits; the rest (the band) is decided on the fp64 logits unless
      // all of it is needed
      const double t = (double)key_value(Tk[r]);  // the k-th largest fp32 logit
      const double e = ErrBound<D>::value * (double)qnorm[bh * nblocks + row] * (double)kmax + 0x1p-100;
      // bounds rounded outwards to fp32: compared with the fp32 logits they
      // keep every block the fp64 bounds would put in the band
      float lo = __double2float_rd(t - 2.0 * e), hi = __double2float_ru(t + 2.0 * e);
      if (!(lo > -INFINITY && hi < INFINITY)) {  // overflow or NaN: decide all in fp64
        lo = -INFINITY;
        hi = INFINITY;
      }
      uint32_t band = 0u;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (key[r][u] == 0u) continue;
        const float L = key_value(key[r][u]);
        if (L > hi)
          taken |= 1u << u;
        else if (L >= lo)
          band |= 1u << u;
      }
      const int need = keep - (int)__reduce_add_sync(kFullMaskScore, (unsigned)__popc(taken));
      const int nband = (int)__reduce_add_sync(kFullMaskScore, (unsigned)__popc(band));
      by_index = false;
      if (nband == need) {
        taken |= band;
      } else {
        double* sv = reinterpret_cast<double*>(shf4) + warp * NK;
        int* sj = reinterpret_cast<int*>(reinterpret_cast<double*>(shf4) + kRegScoreWarps * NK) +
                  warp * NK;
        taken = rank_band64<D, U>(q64 + (bh * nblocks + row) * D, k64 + bh * nblocks * D, band,
                                  need, taken, lane, sv, sj);
      }
    }
    if (by_index) {
      uint32_t tie = 0u;
      unsigned c_gt = 0;
      if constexpr (!CERT) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (key[r][u] > Tk[r]) {
            taken |= 1u << u;
            ++c_gt;
          } else if (key[r][u] == Tk[r]) {
            tie |= 1u << u;
          }
        }
        int eq_left = keep - (int)__reduce_add_sync(kFullMaskScore, c_gt);
#pragma unroll
        for (int u = 0; u < U; ++u) {  // block order: u, then lane
          const bool eq = (tie >> u) & 1u;
          const uint32_t bal = __ballot_sync(kFullMaskScore, eq);
          if (eq && __popc(bal & below) < eq_left) taken |= 1u << u;
          eq_left -= __popc(bal);
        }
      }
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
      double lv[U];
      if constexpr (CERT) {  // the map of the fp64 logits
        row_logits64<D, U>(q64 + (bh * nblocks + row) * D, k64 + bh * nblocks * D, nblocks, lane,
                           lv);
      } else {  // fp32 logits come back from their keys (exactly)
#pragma unroll
        for (int u = 0; u < U; ++u)
          lv[u] = lane + 32 * u < nblocks ? (double)key_value(key[r][u]) : 0.0;
      }
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

// The pooled values in the workspace.  FP32: [fp32 Q | fp32 K].  FP64:
// [fp64 Q | fp64 K][fp32 Q | fp32 K][norms of Q | norms of K].
struct DraftWs {
  const double *q64 = nullptr, *k64 = nullptr;
  const float *q32, *k32, *qn = nullptr, *kn = nullptr;
  DraftWs(const Geometry& g, const void* ws, bool f64) {
    const int64_t n = (int64_t)g.B * g.Hh * g.nblocks;  // units per tensor
    const float* w32 = static_cast<const float*>(ws);
    if (f64) {
      q64 = static_cast<const double*>(ws);
      k64 = q64 + n * g.D;
      w32 = reinterpret_cast<const float*>(q64 + 2 * n * g.D);
      qn = w32 + 2 * n * g.D;
      kn = qn + n;
    }
    q32 = w32;
    k32 = w32 + n * g.D;
  }
};

template <int D, int U>
cudaError_t launch_score_reg(const Geometry& g, const DraftWs& w, int keep, int32_t* row_ptr,
                             int32_t* kv_idx, float* draft_map, cudaStream_t st) {
  using Cfg = RegScoreCfg<U>;
  const bool cert = w.q64 != nullptr;
  auto kern = cert ? draft_score_reg_kernel<D, U, true> : draft_score_reg_kernel<D, U, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Cfg::kSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((g.nblocks + Cfg::kRows - 1) / Cfg::kRows), (unsigned)g.Hh,
                  (unsigned)g.B);
  kern<<<grid, 32 * kRegScoreWarps, Cfg::kSmem, st>>>(w.q32, w.k32, g.Hh, (int)g.nblocks, keep,
                                                       row_ptr, kv_idx, draft_map, w.q64, w.k64,
                                                       w.qn, w.kn);
  return cudaGetLastError();
}

template <int D, typename T>
cudaError_t launch_score_rows(const Geometry& g, const T* qb, const T* kb, int keep,
                              int32_t* row_ptr, int32_t* kv_idx, float* draft_map,
                              cudaStream_t st) {
  const int R = draft_rows_per_cta(g.nblocks, sizeof(T) == 8 ? BSA_DRAFT_FP64 : BSA_DRAFT_FP32);
  const size_t smem = (size_t)(2 * (kScoreThreads / 32) * D + kKeyChunk * (D + 2) +
                               (int64_t)R * g.nblocks) * sizeof(T) +
                      (size_t)R * g.nblocks;
  auto kern = draft_score_topk_kernel<D, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((g.nblocks + R - 1) / R), (unsigned)g.Hh, (unsigned)g.B);
  kern<<<grid, kScoreThreads, smem, st>>>(qb, kb, g.Hh, (int)g.nblocks, R, keep, row_ptr, kv_idx,
                                          draft_map);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_score(const Geometry& g, const DraftWs& w, int keep, int32_t* row_ptr,
                         int32_t* kv_idx, float* draft_map, cudaStream_t st) {
  // rows of up to 512 key blocks: logits in registers
  // (one kernel per 32-block width U: no padded keys beyond the next 32)
  if (g.nblocks <= 512) {
    switch ((g.nblocks + 31) / 32) {
#define BSA_SCORE_U(u) \
  case u:              \
    return launch_score_reg<D, u>(g, w, keep, row_ptr, kv_idx, draft_map, st);
      BSA_SCORE_U(1) BSA_SCORE_U(2) BSA_SCORE_U(3) BSA_SCORE_U(4) BSA_SCORE_U(5) BSA_SCORE_U(6)
      BSA_SCORE_U(7) BSA_SCORE_U(8) BSA_SCORE_U(9) BSA_SCORE_U(10) BSA_SCORE_U(11)
      BSA_SCORE_U(12) BSA_SCORE_U(13) BSA_SCORE_U(14) BSA_SCORE_U(15) BSA_SCORE_U(16)
#undef BSA_SCORE_U
      default:
        break;
    }
  }
  // longer rows: logits in shared memory, in the plan's precision
  if (w.q64)
    return launch_score_rows<D, double>(g, w.q64, w.k64, keep, row_ptr, kv_idx, draft_map, st);
  return launch_score_rows<D, float>(g, w.q32, w.k32, keep, row_ptr, kv_idx, draft_map, st);
}

template <int D>
cudaError_t launch_t(const Geometry& g, const uint32_t* tile_valid, const void* q, const void* k,
                     int keep, int pooling, int precision, bool natural, int32_t* row_ptr,
                     int32_t* kv_idx, float* draft_map, void* ws, cudaStream_t st, uint32_t* amax,
                     bool* amax_recorded) {
  const int use_max = pooling == BSA_POOL_MAX ? 1 : 0;
  const bool f64 = precision == BSA_DRAFT_FP64;
  cudaError_t e = launch_pool<D>(g, tile_valid, q, k, use_max, natural, f64, ws, amax, st);
  if (e != cudaSuccess) return e;
  if (amax_recorded) *amax_recorded = amax != nullptr;
  return launch_score<D>(g, DraftWs(g, ws, f64), keep, row_ptr, kv_idx, draft_map, st);
}

}  // namespace

int draft_rows_per_cta(int64_t nblocks, int precision) {
  // logits + selection flags of R rows within ~150 KB of shared memory; at
  // most two rows per warp of the scoring kernel
  static_assert(2 * (kScoreThreads / 32) >= 16, "two rows per warp");
  const int64_t per = precision == BSA_DRAFT_FP64 ? 9 : 5;
  int64_t R = 16;
  while (R > 1 && R * nblocks * per > 150 * 1024) R >>= 1;
  return (int)R;
}

size_t draft_workspace_bytes(const Geometry& g, int precision) {
  const size_t n = (size_t)g.B * g.Hh * g.nblocks;  // units per tensor
  if (precision == BSA_DRAFT_FP64) return 2 * n * g.D * (sizeof(double) + sizeof(float)) + 2 * n * sizeof(float);
  return 2 * n * g.D * sizeof(float);
}

cudaError_t launch_draft_mask(const Geometry& g, const uint32_t* tile_valid, const void* q,
                              const void* k, int keep, int pooling, int precision,
                              int32_t* row_ptr, int32_t* kv_idx, float* draft_map, void* ws,
                              cudaStream_t st, bool natural, uint32_t* amax, bool* amax_recorded) {
  if (g.D == 128)
    return launch_t<128>(g, tile_valid, q, k, keep, pooling, precision, natural, row_ptr, kv_idx,
                         draft_map, ws, st, amax, amax_recorded);
  return launch_t<64>(g, tile_valid, q, k, keep, pooling, precision, natural, row_ptr, kv_idx,
                      draft_map, ws, st, amax, amax_recorded);
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
// The array is kNoAllocScratchBytes (48 MiB) on every GPU that loads this
// library, held until the process exits; problems whose scratch would exceed
// it (bsa_draft_workspace_bytes) are rejected.  Every call on a device shares the
// one array, so calls whose kernels overlap on the GPU (on different streams,
// or from different host threads) race on it; calls in order on one stream
// are safe.  The array keeps the last call's contents: nothing needs clearing,
// because the pooling kernel writes every element the scoring kernel reads.
// ---------------------------------------------------------------------------
#include <mutex>

namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = 48u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchBytes / sizeof(double)];

// Device address of g_noalloc_scratch on the current device.  Looked up once
// per device, on the first call made with that device current, and cached
// for the life of the process: after cudaDeviceReset the cached address no
// longer names live memory, so the entry point must not be called again in
// that process.
cudaError_t noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
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
  const size_t need = draft_workspace_bytes(g, plan->draft_precision);
  if (need > kNoAllocScratchBytes)
    return set_error(BSA_ERR_UNSUPPORTED,
                     "draft scratch of " + std::to_string(need) +
                         " bytes exceeds the 48 MiB static scratch of bsa_draft_mask_noalloc; "
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
  void* scratch = nullptr;
  e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(scratch)");
  e = launch_draft_mask(g, plan->d_tile_valid, q_slots, k_slots, keep, plan->draft_pooling,
                        plan->draft_precision, row_ptr, kv_idx, draft_map, scratch,
                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask_noalloc launch");
}
