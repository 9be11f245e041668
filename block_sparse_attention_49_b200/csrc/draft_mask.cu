// Draft mask (Draft Attention article: tokens reshaped to [t,h,w]; Q and K
// average-pooled over pool_h x pool_w tiles into a low-resolution draft
// attention map; the map yields a sparse mask that keeps only the important
// block connections, at a stated sparsity; pool_h*pool_w equals the block
// size of the block-sparse attention that follows).
//
// Two kernels, both on the tile-layout slot tensors (each block = one tile):
//  pool:  qbar/kbar[b,h,blk,:] = mean of the block's non-empty slots, fp64.
//         The sum runs sequentially over the block's slots in order (the
//         tile's row-major order) and is divided once by the token count.
//         With max pooling (which the article's authors tried before
//         settling on the average) it is the channel-wise maximum instead,
//         exact in any order.  16-byte loads; HBM bound.
//  score_topk: for a group of query-block rows of one (b, head), the fp64
//         logits L[i][j] = sum_c qbar_i[c]*kbar_j[c] (sequential over c, the
//         product and the sum each rounded, no fused multiply-add), then per
//         row the k largest, ties to the lower j, by k rounds of a warp-wide
//         arg-max; written ascending.  Optionally the draft map
//         softmax_j(L[i][j]/sqrt(D)) as fp32.
// With this fixed evaluation order the selection is reproducible bit for bit
// by any implementation that follows the same order.
#include <cuda_bf16.h>

#include <cfloat>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
constexpr int kKeyChunk = 32;  // key blocks staged in shared memory per step
constexpr int kRegCand = 16;   // top-k candidates per lane held in registers (Nb <= 512)

// One group of D/8 threads per (which, b, h, block); each thread owns 8
// channels.  which = 0: Q, 1: K.
template <int D>
__global__ void __launch_bounds__(kPoolThreads)
    draft_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                      const uint32_t* __restrict__ tile_valid, int Hh, int64_t Npad,
                      int64_t nblocks, int block, int64_t groups_per_tensor, int use_max,
                      double* __restrict__ ws) {
  constexpr int kTPG = D / 8;  // threads per group
  const int64_t gid = ((int64_t)blockIdx.x * kPoolThreads + threadIdx.x) / kTPG;
  const int sub = threadIdx.x % kTPG;
  if (gid >= 2 * groups_per_tensor) return;
  const int which = gid >= groups_per_tensor;
  const int64_t g = gid - which * groups_per_tensor;  // (b*Hh + h)*nblocks + blk
  const int64_t bh = g / nblocks, blk = g - bh * nblocks;
  const uint4* src = (which ? k : q) + ((bh * Npad + blk * block) * (D / 8)) + sub;
  const int64_t s0 = blk * block;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = use_max ? -INFINITY : 0.0;
  int cnt = 0;
  for (int e = 0; e < block; ++e) {
    const int64_t s = s0 + e;
    const uint32_t w = __ldg(tile_valid + (s >> 5));
    if (!((w >> (s & 31)) & 1u)) continue;
    const uint4 v = __ldg(src + (int64_t)e * (D / 8));
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v);
    if (use_max) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(pv[i]);
        acc[2 * i] = fmax(acc[2 * i], (double)f.x);
        acc[2 * i + 1] = fmax(acc[2 * i + 1], (double)f.y);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(pv[i]);
        acc[2 * i] = __dadd_rn(acc[2 * i], (double)f.x);
        acc[2 * i + 1] = __dadd_rn(acc[2 * i + 1], (double)f.y);
      }
    }
    ++cnt;
  }
  double* dst = ws + ((int64_t)which * groups_per_tensor + g) * D + sub * 8;
  const double dc = (double)cnt;
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = cnt ? (use_max ? acc[i] : __ddiv_rn(acc[i], dc)) : 0.0;
}

// The same pooling read straight from the natural layout [B, N, Hh, D]: one
// group of D/8 threads per (which, block, b, h), heads fastest, so the
// groups of a warp read neighbouring 256-byte rows of one token.  The tile's
// tokens inside the grid are visited in row-major (a, then b) order, loads
// eight at a time ahead of the sequential fp64 additions.
template <int D>
__global__ void __launch_bounds__(kPoolThreads)
    draft_pool_nat_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, int B, int Hh,
                          int T, int H, int W, int ph, int pw, int TH, int TW, int64_t nblocks,
                          int64_t groups_per_tensor, int use_max, double* __restrict__ ws) {
  constexpr int kTPG = D / 8;
  constexpr int kAhead = 8;
  const int64_t gid = ((int64_t)blockIdx.x * kPoolThreads + threadIdx.x) / kTPG;
  const int sub = threadIdx.x % kTPG;
  if (gid >= 2 * groups_per_tensor) return;
  const int which = gid >= groups_per_tensor;
  const int64_t gg = gid - which * groups_per_tensor;  // (blk * B + b) * Hh + h
  const int h = (int)(gg % Hh);
  const int64_t rest = gg / Hh;
  const int b = (int)(rest % B);
  const int64_t blk = rest / B;
  const int t = (int)(blk / ((int64_t)TH * TW));
  const int r = (int)(blk - (int64_t)t * TH * TW);
  const int i = r / TW, j = r - (r / TW) * TW;
  const int y0 = i * ph, x0 = j * pw;
  const int hn = min(ph, H - y0), wn = min(pw, W - x0);
  const int64_t N = (int64_t)T * H * W;
  const uint4* src = (which ? k : q) + (((int64_t)b * N + ((int64_t)t * H + y0) * W + x0) * Hh + h) *
                                           (D / 8) + sub;
  const int64_t row_step = (int64_t)Hh * (D / 8);  // one token
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = use_max ? -INFINITY : 0.0;
  for (int a = 0; a < hn; ++a) {
    const uint4* rowp = src + (int64_t)a * W * row_step;
    for (int c0 = 0; c0 < wn; c0 += kAhead) {
      uint4 v[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (c0 + u < wn) v[u] = __ldg(rowp + (int64_t)(c0 + u) * row_step);
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        if (c0 + u >= wn) break;
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
        }
      }
    }
  }
  const int cnt = max(hn, 0) * max(wn, 0);
  double* dst = ws + ((int64_t)which * groups_per_tensor + ((int64_t)b * Hh + h) * nblocks + blk) * D +
                sub * 8;
  const double dc = (double)cnt;
#pragma unroll
  for (int e = 0; e < 8; ++e) dst[e] = cnt ? (use_max ? acc[e] : __ddiv_rn(acc[e], dc)) : 0.0;
}

// Unsigned key with the order of the doubles (-0 and +0 equal; no NaN).
__device__ __forceinline__ uint64_t order_key(double v) {
  const uint64_t b = (uint64_t)__double_as_longlong(v + 0.0);  // -0 + 0 = +0
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// grid: (ceil(nblocks / R), Hh, B); R query rows per CTA.
template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    draft_score_topk_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                            int Hh, int nblocks, int R, int keep, int32_t* __restrict__ row_ptr,
                            int32_t* __restrict__ kv_idx, float* __restrict__ draft_map) {
  constexpr int kWarps = kScoreThreads / 32;
  constexpr int kKStride = D + 2;  // even: 16-byte loads of two channels, no bank conflicts
  extern __shared__ double shd[];
  double* sq = shd;                            // [kWarps][D][2]: rows w and w + kWarps
  double* sk = sq + 2 * kWarps * D;            // [kKeyChunk][kKStride]
  double* sl = sk + kKeyChunk * kKStride;      // [R][nblocks] logits
  uint8_t* sel = reinterpret_cast<uint8_t*>(sl + (int64_t)R * nblocks);  // [R][nblocks]
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * Hh + h;
  const int r0 = blockIdx.x * R;
  const int rows = min(R, nblocks - r0);  // R <= 2 * kWarps
  const double* qb = qbar + (bh * nblocks + r0) * D;
  const double* kb = kbar + bh * nblocks * D;
  // warp w carries rows w and w + kWarps: their values at channel c sit side
  // by side (one broadcast 16-byte load); missing rows read zeros
  for (int i = threadIdx.x; i < 2 * kWarps * D; i += kScoreThreads) {
    const int r = i / D, c = i - r * D;
    sq[((r % kWarps) * D + c) * 2 + r / kWarps] = r < rows ? qb[i] : 0.0;
  }
  for (int i = threadIdx.x; i < rows * nblocks; i += kScoreThreads) sel[i] = 0;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key chunks: the next chunk is loaded into registers while the current
  // one is used, then stored to shared memory (padded stride: no conflicts)
  constexpr int kPer = kKeyChunk * D / kScoreThreads;
  double pre[kPer];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = threadIdx.x + u * kScoreThreads;
      const int jj = idx / D, c = idx - jj * D;
      pre[u] = (j0 + jj < nblocks) ? kb[(int64_t)(j0 + jj) * D + c] : 0.0;
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
      const double2* kk = reinterpret_cast<const double2*>(sk + lane * kKStride);
      const double2* qq = reinterpret_cast<const double2*>(sq) + warp * D;
      double acc_a = 0.0, acc_b = 0.0;
#pragma unroll 4
      for (int c2 = 0; c2 < D / 2; ++c2) {
        const double2 kc = kk[c2];
        const double2 q0 = qq[2 * c2], q1 = qq[2 * c2 + 1];
        acc_a = __dadd_rn(acc_a, __dmul_rn(q0.x, kc.x));
        acc_b = __dadd_rn(acc_b, __dmul_rn(q0.y, kc.x));
        acc_a = __dadd_rn(acc_a, __dmul_rn(q1.x, kc.y));
        acc_b = __dadd_rn(acc_b, __dmul_rn(q1.y, kc.y));
      }
      sl[(int64_t)warp * nblocks + j0 + lane] = acc_a;
      if (warp + kWarps < rows) sl[(int64_t)(warp + kWarps) * nblocks + j0 + lane] = acc_b;
    }
  }
  __syncthreads();

  // top-k per row, one warp per row: k rounds of a warp-wide arg-max (larger
  // logit first, then the lower block index)
  for (int r = warp; r < rows; r += kWarps) {
    const double* L = sl + (int64_t)r * nblocks;
    uint8_t* sr = sel + (int64_t)r * nblocks;
    if (nblocks <= 32 * kRegCand) {
      // candidates j = lane + 32u held in registers as order-preserving
      // 64-bit keys; `avail` marks the ones not yet taken.  A round takes
      // the largest key by three warp reductions (high word, low word among
      // equal high words, lowest index among equal keys).
      uint64_t key[kRegCand];
      uint32_t avail = 0u;
#pragma unroll
      for (int u = 0; u < kRegCand; ++u) {
        const int j = lane + 32 * u;
        key[u] = j < nblocks ? order_key(L[j]) : 0ull;
        if (j < nblocks) avail |= 1u << u;
      }
      const uint32_t start = avail;
      for (int it = 0; it < keep; ++it) {
        uint64_t bk = 0ull;
        int bu = -1;
#pragma unroll
        for (int u = 0; u < kRegCand; ++u)
          if (((avail >> u) & 1u) && (bu < 0 || key[u] > bk)) {
            bk = key[u];
            bu = u;
          }
        const uint32_t hi = bu < 0 ? 0u : (uint32_t)(bk >> 32);
        const uint32_t top_hi = __reduce_max_sync(0xffffffffu, hi);
        const bool at_hi = bu >= 0 && hi == top_hi;
        const uint32_t lo = at_hi ? (uint32_t)bk : 0u;
        const uint32_t top_lo = __reduce_max_sync(0xffffffffu, lo);
        const uint32_t idx = (at_hi && lo == top_lo) ? (uint32_t)(lane + 32 * bu) : 0xffffffffu;
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
        double best = -DBL_MAX;
        int bidx = 0x7fffffff;
        for (int j = lane; j < nblocks; j += 32) {
          if (sr[j]) continue;
          const double v = L[j];
          if (bidx == 0x7fffffff || v > best || (v == best && j < bidx)) {
            best = v;
            bidx = j;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const double ov = __shfl_xor_sync(0xffffffffu, best, o);
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
      for (int j = lane; j < nblocks; j += 32) mx = fmax(mx, L[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const double inv_sqrt_d = 1.0 / sqrt((double)D);
      double sum = 0.0;
      for (int j = lane; j < nblocks; j += 32) sum += exp((L[j] - mx) * inv_sqrt_d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      float* dm = draft_map + grow * nblocks;
      for (int j = lane; j < nblocks; j += 32) dm[j] = (float)(exp((L[j] - mx) * inv_sqrt_d) / sum);
    }
  }
}

template <int D>
cudaError_t launch_t(const Geometry& g, const uint32_t* tile_valid, const void* q, const void* k,
                     int keep, int pooling, bool natural, int32_t* row_ptr, int32_t* kv_idx,
                     float* draft_map, double* ws, cudaStream_t st) {
  const int64_t groups = (int64_t)g.B * g.Hh * g.nblocks;
  const int64_t threads = 2 * groups * (D / 8);
  const unsigned pool_grid = (unsigned)((threads + kPoolThreads - 1) / kPoolThreads);
  const int use_max = pooling == BSA_POOL_MAX ? 1 : 0;
  if (natural)
    draft_pool_nat_kernel<D><<<pool_grid, kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), g.B, g.Hh, g.T, g.H,
        g.W, g.ph, g.pw, g.TH, g.TW, g.nblocks, groups, use_max, ws);
  else
    draft_pool_kernel<D><<<pool_grid, kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), tile_valid, g.Hh,
        g.Npad, g.nblocks, g.block, groups, use_max, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int R = draft_rows_per_cta(g.nblocks);
  const size_t smem = (size_t)(2 * (kScoreThreads / 32) * D + kKeyChunk * (D + 2) +
                               (int64_t)R * g.nblocks) * sizeof(double) +
                      (size_t)R * g.nblocks;
  auto kern = draft_score_topk_kernel<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((g.nblocks + R - 1) / R), (unsigned)g.Hh, (unsigned)g.B);
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
  while (R > 1 && R * nblocks * 9 > 150 * 1024) R >>= 1;
  return (int)R;
}

size_t draft_workspace_bytes(const Geometry& g) {
  return (size_t)2 * g.B * g.Hh * g.nblocks * g.D * sizeof(double);
}

cudaError_t launch_draft_mask(const Geometry& g, const uint32_t* tile_valid, const void* q,
                              const void* k, int keep, int pooling, int32_t* row_ptr,
                              int32_t* kv_idx, float* draft_map, double* ws, cudaStream_t st,
                              bool natural) {
  if (g.D == 128)
    return launch_t<128>(g, tile_valid, q, k, keep, pooling, natural, row_ptr, kv_idx, draft_map,
                         ws, st);
  return launch_t<64>(g, tile_valid, q, k, keep, pooling, natural, row_ptr, kv_idx, draft_map, ws,
                      st);
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

static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchBytes / sizeof(double)];

// Device address of g_noalloc_scratch on the current device.  Looked up once
// per device, on the first call made with that device current.
cudaError_t noalloc_scratch_address(double** out) {
  static std::mutex mu;
  static double* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = reinterpret_cast<double*>(p);
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
  const int keep = (int)((g.nblocks * (100 - sparsity_pct) + 99) / 100);
  if ((int64_t)g.B * g.Hh * g.nblocks * keep >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  double* scratch = nullptr;
  cudaError_t e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(scratch)");
  e = launch_draft_mask(g, plan->d_tile_valid, q_slots, k_slots, keep, plan->draft_pooling, row_ptr,
                        kv_idx, draft_map, scratch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask_noalloc launch");
}
