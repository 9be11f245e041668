// Block-sparse attention on a shared block list, two query tiles per CTA.
//
// What it computes: that of bsa_attn_fwd ("LVSA: Training-Free Sparse
// Attention for Long Video Diffusion", section 2: attention restricted to
// the blocks of the frame set A(t); Draft Attention article: the sparse mask
// guides full-resolution block-sparse attention) for lists shared by every
// (batch, head) with 128-slot blocks: the LVSA block list, or a dense one.
//
// Why: the query blocks of one LVSA frame have identical lists, so two
// neighbouring query tiles can share every K/V tile.  The CTA takes the
// union of the two rows' key blocks; a key tile listed by only one of the
// two rows is masked for the other (at 13 blocks a frame, one pair in
// thirteen straddles two frames).  The pipeline is that of the one-kernel
// LVSA attention: while one query tile's softmax runs, the tensor cores
// work on the other's products.
//
// Roles (12 warps): warp 0 loads both query tiles, then K and V of every
// key tile into 2-deep rings (a K slot is refilled once its last QK is done,
// a V slot after its last PV); warp 1 issues the MMAs in the order PV0(j),
// QK0(j+1), PV1(j), QK1(j+1); warps 4-7 / 8-11 are the softmax of query tile
// 0 / 1, one row per thread, P handed over in two 64-key halves.
// Tensor memory: S0 | S1 | O0 | O1.  Every wait is bounded.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>

#include "attn_common.cuh"
#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 384;
constexpr int kPairMaxTiles = 4096;     // blocks of the plan: a row may name all of them, so
                                        // the union of two rows and the bitmaps fit this

template <int D>
struct PairCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kPanel = kTile * 128;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int NS = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + NS * kTileBytes;
  static constexpr int kOffBar = kOffV + NS * kTileBytes;
  // q_full, k_full[NS], v_full[NS], k_empty[NS], v_empty[NS], s_full[2],
  // p_half[2], p_ready[2], o_final
  static constexpr int kNumBars = 1 + 4 * NS + 2 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffList = kOffMisc + 16;                  // union: (block << 2) | rows
  static constexpr int kOffBits = kOffList + kPairMaxTiles * 4;   // [2][kPairMaxTiles / 32]
  static constexpr int kBytes = kOffBits + 2 * (kPairMaxTiles / 32) * 4;
  static constexpr int kSmem = kBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct PairParams {
  int Hh;
  int64_t Npad, nblocks, ntiles;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  float scale, scale_log2;
  __nv_bfloat16* o;
  float* lse;
  const uint32_t* tile_valid;
  unsigned int* status;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void pair_end_sync() { asm volatile("bar.sync 2, 384;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const PairParams p) {
  using Cfg = PairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + Cfg::NS;
  uint64_t* k_empty = v_full + Cfg::NS;
  uint64_t* v_empty = k_empty + Cfg::NS;
  uint64_t* s_full = v_empty + Cfg::NS;  // [2]
  uint64_t* p_half = s_full + 2;         // [2]
  uint64_t* p_ready = p_half + 2;        // [2]
  uint64_t* o_final = p_ready + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);  // tmem, abort, n, skip
  uint32_t* ulist = reinterpret_cast<uint32_t*>(smem + Cfg::kOffList);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + Cfg::kOffBits);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pr = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh_row = ((int64_t)b * p.Hh + h) * p.Npad;
  const int words = (int)((p.nblocks + 31) >> 5);
  const WaitCtx wc{p.status, reinterpret_cast<volatile int*>(&misc[1]), p.wait_limit_ns};

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < Cfg::NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_half[0], 128);
    mbar_init(&p_half[1], 128);
    mbar_init(&p_ready[0], 128);
    mbar_init(&p_ready[1], 128);
    mbar_init(o_final, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = (*reinterpret_cast<volatile unsigned int*>(p.status) & kStatusTimeout) ? 1u : 0u;
    fence_mbar_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  for (int i = threadIdx.x; i < 2 * words; i += kThreads) bits[(i / words) * (kPairMaxTiles / 32) + i % words] = 0u;
  __syncthreads();
  if (misc[3]) return;
  if (warp == 1) {
    tmem_alloc(&misc[0], 512);
    tmem_relinquish();
  }
  // membership of the two rows' key blocks (query tiles 2 pr and 2 pr + 1)
  const int64_t nnz = p.row_ptr[p.nblocks];
  for (int g = 0; g < 2; ++g) {
    const int64_t qt = 2 * (int64_t)pr + g;
    if (qt >= p.ntiles) continue;
    const int64_t a = p.row_ptr[qt], e = p.row_ptr[qt + 1];
    if (e < a || a < 0 || e > nnz) {
      if (threadIdx.x == 0) atomicOr(p.status, kStatusBadBlocklist);
      continue;
    }
    for (int64_t i = a + threadIdx.x; i < e; i += kThreads) {
      const int c = __ldg(p.col_idx + i);
      if (c >= 0 && (int64_t)c < p.nblocks)
        atomicOr(&bits[g * (kPairMaxTiles / 32) + (c >> 5)], 1u << (c & 31));
      else
        atomicOr(p.status, kStatusBadBlocklist);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // the union in block order, with the rows that list each block
    int cnt = 0;
    bool overflow = false;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t b0 = w < words ? bits[w] : 0u;
      const uint32_t b1 = w < words ? bits[kPairMaxTiles / 32 + w] : 0u;
      const uint32_t u = b0 | b1;
      const int mine = __popc(u);
      int pos = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {  // inclusive prefix sum of the counts
        const int y = __shfl_up_sync(kFullMask, pos, o);
        if (lane >= o) pos += y;
      }
      int at = cnt + pos - mine;
      uint32_t rest = u;
      while (rest) {
        const int bit = __ffs(rest) - 1;
        rest &= rest - 1;
        const uint32_t blk = (uint32_t)(w * 32 + bit);
        const uint32_t rows = ((b0 >> bit) & 1u) | (((b1 >> bit) & 1u) << 1);
        if (at < kPairMaxTiles) ulist[at] = (blk << 2) | rows;
        else overflow = true;
        ++at;
      }
      cnt += __shfl_sync(kFullMask, pos, 31);
    }
    if (__any_sync(kFullMask, overflow) && lane == 0) atomicOr(p.status, kStatusBadBlocklist);
    if (lane == 0) misc[2] = (uint32_t)min(cnt, kPairMaxTiles);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];
  const int n = (int)misc[2];

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
    if (warp == 0 && n > 0) {
      // -------------------------------------------------------- TMA producer
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, 2 * Cfg::kTileBytes);
        for (int g = 0; g < 2; ++g)
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_2d(sQ + g * Cfg::kTileBytes + c * Cfg::kPanel, &tmq, q_full, c * 64,
                        (int)(bh_row + (2 * (int64_t)pr + g) * kTile));
      }
      __syncwarp();
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % Cfg::NS;
        const uint32_t par = ((j / Cfg::NS) & 1) ^ 1;
        const int krow = (int)(bh_row + (int64_t)(ulist[j] >> 2) * kTile);
        if (!__all_sync(kFullMask, bounded_wait(&k_empty[st], par, wc))) break;
        if (elect_one()) {
          uint8_t* sK = smem + Cfg::kOffK + st * Cfg::kTileBytes;
          mbar_arrive_expect_tx(&k_full[st], Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c) tma_load_2d(sK + c * Cfg::kPanel, &tmk, &k_full[st], c * 64, krow);
        }
        __syncwarp();
        issued_k = j + 1;
        if (!__all_sync(kFullMask, bounded_wait(&v_empty[st], par, wc))) break;
        if (elect_one()) {
          uint8_t* sV = smem + Cfg::kOffV + st * Cfg::kTileBytes;
          mbar_arrive_expect_tx(&v_full[st], Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c) tma_load_2d(sV + c * Cfg::kPanel, &tmv, &v_full[st], c * 64, krow);
        }
        __syncwarp();
        issued_v = j + 1;
      }
      if (*wc.abort) {
        // leave no copy in flight (bounded waits that ignore the abort flag)
        volatile int no_abort = 0;
        const WaitCtx drain{p.status, &no_abort, p.wait_limit_ns};
        bounded_wait(q_full, 0, drain);
        for (int j = max(0, issued_k - Cfg::NS); j < issued_k; ++j)
          bounded_wait(&k_full[j % Cfg::NS], (j / Cfg::NS) & 1, drain);
        for (int j = max(0, issued_v - Cfg::NS); j < issued_v; ++j)
          bounded_wait(&v_full[j % Cfg::NS], (j / Cfg::NS) & 1, drain);
      }
      __syncwarp();
    } else if (warp == 1 && n > 0) {
      // -------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
      constexpr uint32_t dhi = sdesc_sw128_hi(1024);
      const uint32_t q_lo = sdesc_sw128_lo(smem_u32(sQ), 16);
      const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + Cfg::kOffK), 16);
      const uint32_t v_lo = sdesc_sw128_lo(smem_u32(smem + Cfg::kOffV), Cfg::kPanel);
      auto issue_qk = [&](int g, int st) {
        const uint32_t dst = tbase + g * 128;
        const uint32_t qd = q_lo + ((g * Cfg::kTileBytes) >> 4);
        const uint32_t kd = k_lo + ((st * Cfg::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * Cfg::kPanel + (kk & 3) * 32) >> 4;
            mma_ss(dst, sdesc_join(dhi, qd + off), sdesc_join(dhi, kd + off), idesc_qk, kk > 0);
          }
          mma_commit(&s_full[g]);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int g, int st, int half, uint32_t acc) {
        const uint32_t dst = tbase + 256 + g * 128, pa = tbase + g * 128 + 64 + half * 32;
        const uint32_t vd = v_lo + ((st * Cfg::kTileBytes + half * 8192) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(dst, pa + kk * 8, sdesc_join(dhi, vd + kk * (2048 >> 4)), idesc_pv,
                   (acc | (uint32_t)half | (uint32_t)kk) != 0);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) mma_commit(bar);
        __syncwarp();
      };
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(kFullMask, bounded_wait(bar, parity, wc));
      };
      bool alive = wait(q_full, 0) && wait(&k_full[0], 0);
      if (alive) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        commit(&k_empty[0]);
      }
      for (int j = 0; alive && j < n; ++j) {
        const int st = j % Cfg::NS, st1 = (j + 1) % Cfg::NS;
        if (!wait(&p_half[0], j & 1) || !wait(&v_full[st], (j / Cfg::NS) & 1)) break;
        tc_fence_after();
        issue_pv(0, st, 0, j > 0);
        if (!wait(&p_ready[0], j & 1)) break;
        tc_fence_after();
        issue_pv(0, st, 1, 1);
        if (j + 1 < n) {
          if (!wait(&k_full[st1], ((j + 1) / Cfg::NS) & 1)) break;
          tc_fence_after();
          issue_qk(0, st1);
        }
        if (!wait(&p_half[1], j & 1)) break;
        tc_fence_after();
        issue_pv(1, st, 0, j > 0);
        if (!wait(&p_ready[1], j & 1)) break;
        tc_fence_after();
        issue_pv(1, st, 1, 1);
        commit(&v_empty[st]);
        if (j + 1 < n) {
          issue_qk(1, st1);
          commit(&k_empty[st1]);
        }
      }
      commit(o_final);
    }
    pair_end_sync();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tbase, 512);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    // ---------------------------------------------------------- softmax
    const int g = (warp >= 8) ? 1 : 0;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + g * 128 + lane_off;
    const uint32_t tO = tbase + 256 + g * 128 + lane_off;
    const int64_t qt = 2 * (int64_t)pr + g;
    const bool tile_ok = qt < p.ntiles;
    const float sl2 = p.scale_log2;
    const float thr = 8.0f / sl2;
    RowState st;
    bool alive = true;
    for (int j = 0; j < n; ++j) {
      // keys of tile j: the block's non-empty slots if this row lists the block
      uint32_t vm[4] = {0u, 0u, 0u, 0u};
      const uint32_t e = ulist[j];
      if (tile_ok && ((e >> g) & 1u)) {
        const uint4 tv = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + (e >> 2));
        vm[0] = tv.x;
        vm[1] = tv.y;
        vm[2] = tv.z;
        vm[3] = tv.w;
      }
      if (!__all_sync(kFullMask, bounded_wait(&s_full[g], j & 1, wc))) {
        alive = false;
        break;
      }
      tc_fence_after();
      float s[128];
      {
        uint32_t r128[128];
        tmem_ld128(tS, r128);
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(r128[i]);
      }
      float corr;
      uint64_t neg_ms2;
      const bool need = softmax_max(s, vm, st, sl2, thr, corr, neg_ms2);
      if (j > 0 && __any_sync(kFullMask, need)) tmem_scale<D>(tO, corr);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      {
        uint32_t pk[32];
        softmax_exp<0, 64>(s, sl2, neg_ms2, pk, acc);
        tmem_st32(tS + 64, pk);
      }
      tc_fence_before();
      mbar_arrive(&p_half[g]);
      {
        uint32_t pk[32];
        softmax_exp<64, 64>(s, sl2, neg_ms2, pk, acc);
        tmem_st32(tS + 96, pk);
      }
      softmax_sum(st, acc);
      tc_fence_before();
      mbar_arrive(&p_ready[g]);
    }
    if (alive && n > 0) {
      alive = __all_sync(kFullMask, bounded_wait(o_final, 0, wc));
      tc_fence_after();
    }
    // O and LSE of the slot rows; rows of empty slots get 0 and -inf
    uint32_t qmask = 0u;
    if (tile_ok) {
      const uint4 tq = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + qt);
      qmask = (row < 32) ? tq.x : (row < 64) ? tq.y : (row < 96) ? tq.z : tq.w;
    }
    const bool qvalid = (qmask >> (row & 31)) & 1u;
    const bool has = alive && n > 0 && qvalid && st.l > 0.f;
    const float inv_l = has ? 1.f / st.l : 0.f;
    const int64_t orow = bh_row + qt * kTile + row;
    uint4* dst = reinterpret_cast<uint4*>(p.o + orow * D);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o32[32];
      if (alive && n > 0) {
        tmem_ld32(tO + c * 32, o32);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o32[i] = 0u;
      }
      uint32_t w16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w16[i] = pack_bf16x2(has ? __uint_as_float(o32[2 * i]) * inv_l : 0.f,
                             has ? __uint_as_float(o32[2 * i + 1]) * inv_l : 0.f);
      if (tile_ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[c * 4 + i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
      }
    }
    if (tile_ok && p.lse) p.lse[orow] = has ? st.m * p.scale + logf(st.l) : -INFINITY;
    tc_fence_before();
    pair_end_sync();
  }
}

PFN_cuTensorMapEncodeTiled_v12000 pair_encode_fn() {
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

// Slot layout [rows, D] bf16 row-major, 64 x 128 boxes, 128-byte swizzle.
bool make_pair_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int D) {
  auto fn = pair_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_pair_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const PairParams& p, dim3 grid, cudaStream_t st) {
  auto kern = attn_pair_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, PairCfg<D>::kSmem, st>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

bool attn_pair_applies(const Geometry& g, int per_head) {
  // a row may name every block: the union of two rows must fit the list
  return !per_head && g.block == kTile && g.nblocks <= kPairMaxTiles;
}

bsa_status launch_attn_pair(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                            const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                            float* lse, cudaStream_t st) {
  const Geometry& g = plan.g;
  const int64_t rows = (int64_t)g.B * g.Hh * g.Npad;
  if (rows >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "B*Hh*Npad must be < 2^31");
  CUtensorMap tq, tk, tv;
  if (!make_pair_tmap(&tq, q, rows, g.D) || !make_pair_tmap(&tk, k, rows, g.D) ||
      !make_pair_tmap(&tv, v, rows, g.D))
    return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  PairParams p;
  p.Hh = g.Hh;
  p.Npad = g.Npad;
  p.nblocks = g.nblocks;
  p.ntiles = g.ntiles;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.tile_valid = plan.d_tile_valid;
  p.status = plan.d_status;
  p.wait_limit_ns = plan.wait_limit_ns;
  const dim3 grid((unsigned)((g.ntiles + 1) / 2), (unsigned)g.Hh, (unsigned)g.B);
  const cudaError_t e = g.D == 128 ? launch_pair_t<128>(tq, tk, tv, p, grid, st)
                                   : launch_pair_t<64>(tq, tk, tv, p, grid, st);
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "paired attention launch");
}

}  // namespace bsa
