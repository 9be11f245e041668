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
#include <cudaTypedefs.h>

#include <algorithm>
#include <cfloat>

#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
constexpr int kKeyChunk = 32;  // key blocks staged in shared memory per step
constexpr int kRegCand = 16;   // top-k candidates per lane held in registers (Nb <= 512)
constexpr unsigned kFullMaskScore = 0xffffffffu;

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

// ---------------------------------------------------------------------------
// Pooling fed by TMA (tiles of up to 256 tokens): a persistent CTA per SM.
// Warp 0 streams units - (Q or K, tile, batch, head, 64-channel chunk) - into
// a ring of shared-memory stages with one tensor-map load each; warps 1..4
// take the units in turn, each lane summing two channels over the tile's
// tokens in row-major order straight out of shared memory.  The deep ring
// keeps many loads in flight per SM without holding them in registers, so
// the pass runs at the memory's rate at any number of heads.
//   natural layout: 5-D map {D, Hh, W, H, B*T}, box {64, 1, pw, ph, 1} (one
//     pooling tile of one head; parts past the grid read as zero and are
//     skipped);
//   slot layout: 2-D map {D, B*Hh*Npad}, box {64, block} (one block; empty
//     slots skipped by the plan's validity bits).
// Optionally records max |x| per (Q or K, batch, head) for the e4m3 scales.
// ---------------------------------------------------------------------------
constexpr int kPoolTmaConsumers = 4;
constexpr int kPoolTmaThreads = 32 * (1 + kPoolTmaConsumers);
constexpr int kPoolTmaMaxStages = 8;
constexpr int kPoolTmaSmemBudget = 160 * 1024;

struct PoolTmaParams {
  int B, Hh, T, H, W, ph, pw, TH, TW;
  int64_t nblocks, Npad;
  int rows;          // box rows: pw * ph (natural) or the block size (slots)
  int nchunk;        // D / 64
  int stages;
  int64_t units;     // 2 * nblocks * B * Hh * nchunk
  int use_max;
  const uint32_t* tile_valid;
  uint32_t* amax;    // [3][B][Hh] float bits, or null
  double* ws;
  unsigned int* status;
  uint64_t wait_limit_ns;
};

template <int D, bool NAT>
__global__ void __launch_bounds__(kPoolTmaThreads, 1)
    draft_pool_tma_kernel(const __grid_constant__ CUtensorMap tmq,
                          const __grid_constant__ CUtensorMap tmk, const PoolTmaParams p) {
  extern __shared__ uint8_t pool_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pool_smem_raw) + 127) &
                                             ~uintptr_t(127));
  const int stage_bytes = p.rows * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * stage_bytes);
  uint64_t* empty = full + kPoolTmaMaxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kPoolTmaMaxStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(p.status) & kStatusTimeout) ? 1 : 0;
    fence_mbar_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
  }
  __syncthreads();
  if (*abort_flag) return;
  const WaitCtx wc{p.status, abort_flag, p.wait_limit_ns};
  const int64_t per_which = p.units / 2;
  const int64_t nbh = (int64_t)p.B * p.Hh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int64_t k = 0, issued = 0;
    for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x, ++k) {
      const int st = (int)(k % p.stages);
      const uint32_t par = (uint32_t)((k / p.stages) & 1) ^ 1u;
      if (!__all_sync(kFullMaskScore, bounded_wait(&empty[st], par, wc))) break;
      const int which = u >= per_which;
      const int64_t r = u - which * per_which;
      const int chunk = (int)(r % p.nchunk);
      const int64_t r2 = r / p.nchunk;
      if (elect_one()) {
        const CUtensorMap* m = which ? &tmk : &tmq;
        mbar_arrive_expect_tx(&full[st], (uint32_t)stage_bytes);
        uint8_t* dst = smem + (size_t)st * stage_bytes;
        if (NAT) {
          // r2 = (blk * B + b) * Hh + h
          const int h = (int)(r2 % p.Hh);
          const int64_t r3 = r2 / p.Hh;
          const int b = (int)(r3 % p.B);
          const int64_t blk = r3 / p.B;
          const int t = (int)(blk / ((int64_t)p.TH * p.TW));
          const int rr = (int)(blk - (int64_t)t * p.TH * p.TW);
          const int i = rr / p.TW, j = rr - (rr / p.TW) * p.TW;
          tma_load_5d(dst, m, &full[st], chunk * 64, h, j * p.pw, i * p.ph, b * p.T + t);
        } else {
          // r2 = (b * Hh + h) * nblocks + blk
          const int64_t bh = r2 / p.nblocks, blk = r2 - bh * p.nblocks;
          tma_load_2d(dst, m, &full[st], chunk * 64, (int)(bh * p.Npad + blk * p.rows));
        }
      }
      __syncwarp();
      issued = k + 1;
    }
    if (*wc.abort) {
      // leave no copy in flight: wait (bounded, ignoring the abort flag) for
      // the loads still owned by the ring
      volatile int no_abort = 0;
      const WaitCtx drain{p.status, &no_abort, p.wait_limit_ns};
      for (int64_t q = std::max<int64_t>(0, issued - p.stages); q < issued; ++q)
        bounded_wait(&full[q % p.stages], (uint32_t)((q / p.stages) & 1), drain);
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  int64_t k = cw;
  for (int64_t u = blockIdx.x + (int64_t)cw * gridDim.x; u < p.units;
       u += (int64_t)kPoolTmaConsumers * gridDim.x, k += kPoolTmaConsumers) {
    const int st = (int)(k % p.stages);
    if (!__all_sync(kFullMaskScore, bounded_wait(&full[st], (uint32_t)((k / p.stages) & 1), wc)))
      return;
    const int which = u >= per_which;
    const int64_t r = u - which * per_which;
    const int chunk = (int)(r % p.nchunk);
    const int64_t r2 = r / p.nchunk;
    int b, h;
    int64_t blk;
    int hn, wn;
    if (NAT) {
      h = (int)(r2 % p.Hh);
      const int64_t r3 = r2 / p.Hh;
      b = (int)(r3 % p.B);
      blk = r3 / p.B;
      const int rr = (int)(blk % ((int64_t)p.TH * p.TW));
      const int i = rr / p.TW, j = rr - (rr / p.TW) * p.TW;
      hn = min(p.ph, p.H - i * p.ph);
      wn = min(p.pw, p.W - j * p.pw);
    } else {
      const int64_t bh = r2 / p.nblocks;
      blk = r2 - bh * p.nblocks;
      b = (int)(bh / p.Hh);
      h = (int)(bh - (int64_t)b * p.Hh);
      hn = 1;
      wn = p.rows;
    }
    const uint32_t* src = reinterpret_cast<const uint32_t*>(smem + (size_t)st * stage_bytes) + lane;
    const bool use_max = p.use_max != 0;
    double a0 = use_max ? -INFINITY : 0.0, a1 = a0;
    float mabs = 0.f;
    int cnt = 0;
    const int64_t s0 = blk * p.rows;  // first slot (slot layout)
    for (int a = 0; a < hn; ++a) {
      for (int c = 0; c < wn; ++c) {
        const int e = a * p.pw * (NAT ? 1 : 0) + c;
        if (!NAT) {
          const int64_t sl = s0 + c;
          if (!((__ldg(p.tile_valid + (sl >> 5)) >> (sl & 31)) & 1u)) continue;
        }
        const uint32_t v = src[e * 32];
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
        if (use_max) {
          a0 = fmax(a0, (double)f.x);
          a1 = fmax(a1, (double)f.y);
        } else {
          a0 = __dadd_rn(a0, (double)f.x);
          a1 = __dadd_rn(a1, (double)f.y);
        }
        mabs = fmaxf(mabs, fmaxf(fabsf(f.x), fabsf(f.y)));
        ++cnt;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    const double dc = (double)cnt;
    double2 out;
    out.x = cnt ? (use_max ? a0 : __ddiv_rn(a0, dc)) : 0.0;
    out.y = cnt ? (use_max ? a1 : __ddiv_rn(a1, dc)) : 0.0;
    const int64_t gidx = (int64_t)which * nbh * p.nblocks + ((int64_t)b * p.Hh + h) * p.nblocks + blk;
    reinterpret_cast<double2*>(p.ws + gidx * D + chunk * 64)[lane] = out;
    if (p.amax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mabs = fmaxf(mabs, __shfl_xor_sync(kFullMaskScore, mabs, o));
      if (lane == 0) atomicMax(p.amax + ((int64_t)which * p.B + b) * p.Hh + h, __float_as_uint(mabs));
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 pool_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Unswizzled maps with 64-channel boxes: one pooling tile of one head
// (natural layout) or one block of slots.
bool make_pool_tmap(CUtensorMap* m, const void* ptr, const Geometry& g, bool natural) {
  auto fn = pool_encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  if (natural) {
    const cuuint64_t row = (cuuint64_t)g.Hh * g.D * 2;
    cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.Hh, (cuuint64_t)g.W, (cuuint64_t)g.H,
                          (cuuint64_t)g.B * g.T};
    cuuint64_t strides[4] = {(cuuint64_t)g.D * 2, row, row * g.W, row * g.W * g.H};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)g.pw, (cuuint32_t)g.ph, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t dims[2] = {(cuuint64_t)g.D, (cuuint64_t)g.B * g.Hh * g.Npad};
  cuuint64_t strides[1] = {(cuuint64_t)g.D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)g.block};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int n[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    n[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0
                 ? v
                 : 148;
  }
  return n[dev];
}

// TMA pooling applies when a unit (box) is at most 256 token rows and the
// 5-D / 2-D maps can address the tensors.
bool pool_tma_applies(const Geometry& g, bool natural) {
  const int rows = natural ? g.ph * g.pw : g.block;
  if (rows < 1 || rows > 256 || (g.D % 64) != 0) return false;
  if (natural) return g.pw <= 256 && g.ph <= 256;
  return (int64_t)g.B * g.Hh * g.Npad < (1ll << 31);
}

template <int D>
cudaError_t launch_pool_tma(const Geometry& g, const uint32_t* tile_valid, const void* q,
                            const void* k, int use_max, bool natural, double* ws, uint32_t* amax,
                            unsigned int* status, uint64_t wait_limit_ns, cudaStream_t st) {
  CUtensorMap tq, tk;
  if (!make_pool_tmap(&tq, q, g, natural) || !make_pool_tmap(&tk, k, g, natural))
    return cudaErrorInvalidValue;
  PoolTmaParams p;
  p.B = g.B;
  p.Hh = g.Hh;
  p.T = g.T;
  p.H = g.H;
  p.W = g.W;
  p.ph = g.ph;
  p.pw = g.pw;
  p.TH = g.TH;
  p.TW = g.TW;
  p.nblocks = g.nblocks;
  p.Npad = g.Npad;
  p.rows = natural ? g.ph * g.pw : g.block;
  p.nchunk = D / 64;
  const int stage_bytes = p.rows * 128;
  p.stages = std::max(2, std::min(kPoolTmaMaxStages, kPoolTmaSmemBudget / stage_bytes));
  p.units = 2 * g.nblocks * g.B * g.Hh * p.nchunk;
  p.use_max = use_max;
  p.tile_valid = tile_valid;
  p.amax = amax;
  p.ws = ws;
  p.status = status;
  p.wait_limit_ns = wait_limit_ns;
  const size_t smem = 128 + (size_t)p.stages * stage_bytes + 2 * kPoolTmaMaxStages * 8 + 16;
  auto kern = natural ? draft_pool_tma_kernel<D, true> : draft_pool_tma_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(p.units, sm_count());
  kern<<<(unsigned)grid, kPoolTmaThreads, smem, st>>>(tq, tk, p);
  return cudaGetLastError();
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

// ---------------------------------------------------------------------------
// Scoring with the logits in registers (up to 512 key blocks per row).
//
// A warp owns R whole query-block rows; lane l accumulates the logits of key
// blocks j = l + 32u (u < U) of each row, so a row's top-k runs straight out
// of registers and no logit ever goes to shared memory.  The CTA's 8 warps
// share the pooled keys, staged CK channels at a time (transposed to
// [channel][key], so a lane's loads are conflict-free) in a two-stage
// cp.async ring; the pooled query values are broadcast reads.  Every logit
// is still the sequential multiply-then-add chain over c = 0..D-1, each
// operation rounded: only the loop order around the chains changes.
// ---------------------------------------------------------------------------
constexpr int kRegScoreWarps = 8;
constexpr int kRegScoreCK = 8;  // channels per stage

__device__ __forceinline__ void cp_async8(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 8 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int U>
struct RegScoreCfg {
  static constexpr int R = U <= 12 ? 4 : 2;            // rows per warp
  static constexpr int kRows = R * kRegScoreWarps;     // rows per CTA
  static constexpr int NK = 32 * U;                    // keys, padded
  static constexpr int kStageK = kRegScoreCK * NK;     // doubles per K stage
  static constexpr int kStageQ = kRegScoreCK * kRows;  // doubles per Q stage
  static constexpr size_t kSmem = 2 * (size_t)(kStageK + kStageQ) * sizeof(double);
};

// grid: (ceil(nblocks / kRows), Hh, B)
template <int D, int U>
__global__ void __launch_bounds__(32 * kRegScoreWarps, 2)
    draft_score_reg_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                           int Hh, int nblocks, int keep, int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ kv_idx, float* __restrict__ draft_map) {
  using Cfg = RegScoreCfg<U>;
  constexpr int R = Cfg::R, CK = kRegScoreCK, NK = Cfg::NK;
  constexpr int kThreads = 32 * kRegScoreWarps;
  extern __shared__ double shd[];
  double* sK = shd;                   // [2][CK][NK]
  double* sQ = shd + 2 * Cfg::kStageK;  // [2][CK][kRows]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * Hh + h;
  const int r0 = blockIdx.x * Cfg::kRows;
  const double* qb = qbar + bh * nblocks * D;
  const double* kb = kbar + bh * nblocks * D;

  // stage `st` <- channels [c0, c0 + CK): keys transposed, rows transposed;
  // entries past the grid are zero-filled (a valid source address is still
  // passed: the copy reads 0 bytes from it)
  auto issue = [&](int st, int c0) {
    double* dk = sK + st * Cfg::kStageK;
    for (int i = threadIdx.x; i < Cfg::kStageK; i += kThreads) {
      const int j = i / CK, c = i - j * CK;
      const bool ok = j < nblocks;
      cp_async8(dk + c * NK + j, kb + (int64_t)(ok ? j : 0) * D + c0 + c, ok);
    }
    double* dq = sQ + st * Cfg::kStageQ;
    for (int i = threadIdx.x; i < Cfg::kStageQ; i += kThreads) {
      const int r = i / CK, c = i - r * CK;
      const bool ok = r0 + r < nblocks;
      cp_async8(dq + c * Cfg::kRows + r, qb + (int64_t)(ok ? r0 + r : 0) * D + c0 + c, ok);
    }
    cp_async_commit();
  };

  double acc[R][U];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int u = 0; u < U; ++u) acc[r][u] = 0.0;

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
    const double* ck = sK + (cs & 1) * Cfg::kStageK + lane;
    const double* cq = sQ + (cs & 1) * Cfg::kStageQ + warp * R;
#pragma unroll
    for (int c = 0; c < CK; ++c) {
      double qv[R];
#pragma unroll
      for (int r = 0; r < R; ++r) qv[r] = cq[c * Cfg::kRows + r];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const double kv = ck[c * NK + 32 * u];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][u] = __dadd_rn(acc[r][u], __dmul_rn(qv[r], kv));
      }
    }
    __syncthreads();  // the next issue() overwrites this stage
  }

  // top-k of each row: k rounds of a warp-wide arg-max over order-preserving
  // 64-bit keys (larger logit first, then the lower block index)
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int row = r0 + warp * R + r;
    if (row >= nblocks) break;  // warp-uniform
    uint64_t key[U];
    uint32_t avail = 0u;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = lane + 32 * u;
      key[u] = order_key(acc[r][u]);
      if (j < nblocks) avail |= 1u << u;
    }
    const uint32_t start = avail;
    for (int it = 0; it < keep; ++it) {
      uint64_t bk = 0ull;
      int bu = -1;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (((avail >> u) & 1u) && (bu < 0 || key[u] > bk)) {
          bk = key[u];
          bu = u;
        }
      const uint32_t hi = bu < 0 ? 0u : (uint32_t)(bk >> 32);
      const uint32_t top_hi = __reduce_max_sync(kFullMaskScore, hi);
      const bool at_hi = bu >= 0 && hi == top_hi;
      const uint32_t lo = at_hi ? (uint32_t)bk : 0u;
      const uint32_t top_lo = __reduce_max_sync(kFullMaskScore, lo);
      const uint32_t idx = (at_hi && lo == top_lo) ? (uint32_t)(lane + 32 * bu) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(kFullMaskScore, idx);
      if (win != 0xffffffffu && (int)(win & 31u) == lane) avail &= ~(1u << (win >> 5));
    }
    const uint32_t taken = start & ~avail;
    // ascending output: j = 32u + lane grows with (u, lane)
    const int64_t grow = bh * nblocks + row;
    int32_t* out = kv_idx + grow * keep;
    int pos = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool on = (taken >> u) & 1u;
      const uint32_t bal = __ballot_sync(kFullMaskScore, on);
      if (on) {
        const int at = pos + __popc(bal & ((1u << lane) - 1u));
        if (at < keep) out[at] = lane + 32 * u;
      }
      pos += __popc(bal);
    }
    if (row_ptr && lane == 0) {
      row_ptr[grow] = (int32_t)(grow * keep);
      if (grow == (int64_t)gridDim.z * Hh * nblocks - 1) row_ptr[grow + 1] = (int32_t)((grow + 1) * keep);
    }
    if (draft_map) {
      double mx = -DBL_MAX;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks) mx = fmax(mx, acc[r][u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFullMaskScore, mx, o));
      const double inv_sqrt_d = 1.0 / sqrt((double)D);
      double sum = 0.0;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks) sum += exp((acc[r][u] - mx) * inv_sqrt_d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFullMaskScore, sum, o);
      float* dm = draft_map + grow * nblocks;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (lane + 32 * u < nblocks)
          dm[lane + 32 * u] = (float)(exp((acc[r][u] - mx) * inv_sqrt_d) / sum);
    }
  }
}

template <int D, int U>
cudaError_t launch_score_reg(const Geometry& g, const double* ws, int keep, int32_t* row_ptr,
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
                     float* draft_map, double* ws, unsigned int* status, uint64_t wait_limit_ns,
                     cudaStream_t st, uint32_t* amax, bool* amax_recorded) {
  const int64_t groups = (int64_t)g.B * g.Hh * g.nblocks;
  const int64_t threads = 2 * groups * (D / 8);
  const unsigned pool_grid = (unsigned)((threads + kPoolThreads - 1) / kPoolThreads);
  const int use_max = pooling == BSA_POOL_MAX ? 1 : 0;
  if (amax_recorded) *amax_recorded = false;
  if (pool_tma_applies(g, natural)) {
    cudaError_t e0 = launch_pool_tma<D>(g, tile_valid, q, k, use_max, natural, ws, amax, status,
                                        wait_limit_ns, st);
    if (e0 != cudaSuccess) return e0;
    if (amax_recorded) *amax_recorded = amax != nullptr;
  } else if (natural)
    draft_pool_nat_kernel<D><<<pool_grid, kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), g.B, g.Hh, g.T, g.H,
        g.W, g.ph, g.pw, g.TH, g.TW, g.nblocks, groups, use_max, ws);
  else
    draft_pool_kernel<D><<<pool_grid, kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), tile_valid, g.Hh,
        g.Npad, g.nblocks, g.block, groups, use_max, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // rows of up to 512 key blocks: logits in registers
  if (g.nblocks <= 128) return launch_score_reg<D, 4>(g, ws, keep, row_ptr, kv_idx, draft_map, st);
  if (g.nblocks <= 256) return launch_score_reg<D, 8>(g, ws, keep, row_ptr, kv_idx, draft_map, st);
  if (g.nblocks <= 384) return launch_score_reg<D, 12>(g, ws, keep, row_ptr, kv_idx, draft_map, st);
  if (g.nblocks <= 512) return launch_score_reg<D, 16>(g, ws, keep, row_ptr, kv_idx, draft_map, st);
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
                              int32_t* kv_idx, float* draft_map, double* ws, unsigned int* status,
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

static __device__ __align__(256) double g_noalloc_scratch[kNoAllocScratchBytes / sizeof(double)];

// Device address of g_noalloc_scratch on the current device.  Looked up once
// per device, on the first call made with that device current, and cached
// for the life of the process: after cudaDeviceReset the cached address no
// longer names live memory, so the entry point must not be called again in
// that process.
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
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev != plan->device)
    return set_error(BSA_ERR_INVALID_ARG,
                     "the current device is not the plan's: the static scratch of one device "
                     "cannot serve a plan of another");
  double* scratch = nullptr;
  e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(scratch)");
  e = launch_draft_mask(g, plan->d_tile_valid, q_slots, k_slots, keep, plan->draft_pooling, row_ptr,
                        kv_idx, draft_map, scratch, plan->d_status, plan->wait_limit_ns,
                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask_noalloc launch");
}
