// LVSA attention in one kernel, on the natural token layout.
//
// What it computes ("LVSA: Training-Free Sparse Attention for Long Video
// Diffusion", section 2 "Core mechanism"): every query token of frame t
// attends, with softmax(scale * q.k), exactly the key tokens of the frames in
// A(t) = G_s U W(t) - rotating anchors G_s = {f : (f - s) mod T_per = 0} and
// a window around t grown t+1, t-1, t+2, ... past the frames already present
// until |A(t)| = C (or a variant chosen on the plan: fixed-grid or no
// anchors, alternating window growth).  The result equals bsa_lvsa_mask +
// bsa_reorder_fwd + bsa_attn_fwd + bsa_reorder_inv; the reorder of the Draft
// Attention article is fused into the tile loads (a 3-D tensor map reads
// [B*N, Hh, D] rows of one head directly), so no padded copy of Q, K, V or O
// is ever made.
//
// Work unit (one CTA, 12 warps): 256 consecutive query tokens of one
// (b, head) = two 128-row query tiles that share every key tile.
//  * set-up: A(t) for the (at most 8) frames of the 256 queries, as bitmaps
//    over frames; their union U; the key tiles = 128-token pieces of each run
//    of consecutive frames of U.  Membership uses a closed form: a frame f
//    outside G_s U {t} joins iff fewer than C - |G_s U {t}| such frames come
//    before it in the growth order; anchors in a range are counted
//    arithmetically (they are periodic).
//  * warp 0: TMA producer (both query tiles, then K and V of every key tile
//    into 2-deep rings; a K slot is refilled as soon as its last QK product
//    is done, a V slot after its last PV product).  warp 1: MMA issuer.
//    warp 2: key masks - for each key tile and each query frame of the CTA,
//    the rows whose frame is in that frame's A(t), computed a ring of tiles
//    ahead (once per CTA instead of once per softmax warp).
//    warps 4-7 / 8-11: softmax of query tile 0 / 1, one row per thread,
//    masking keys whose frame is not in the row's own A(t).
//  * tensor memory: S0 | S1 | O0 | O1; P aliases the upper half of its S.
//    MMA order per key tile j: PV0(j), QK0(j+1), PV1(j), QK1(j+1), so the
//    tensor cores run one tile's products while the other tile's softmax runs.
//    A softmax group hands P over in two 64-key halves: the PV product of the
//    first half runs while the exponentials of the second are computed.
// Every wait is bounded (see bounded_wait).
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "attn_common.cuh"
#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr int kTile = 128;
constexpr int kPair = 2 * kTile;
constexpr int kThreads = 384;
constexpr int kMaxRowFrames = 8;   // frames a 256-token query pair may touch
constexpr int kMaxFrames = 4096;
constexpr int kSetWords = kMaxFrames / 32;
constexpr int kMaxRuns = 1024;     // runs of consecutive frames in a query pair's union
constexpr int kMaskRing = 16;      // key tiles whose row masks are computed ahead

template <int D>
struct LvsaCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kPanel = kTile * 128;
  static constexpr int kQBytes = kTile * D * 2;
  static constexpr int kKVBytes = kTile * D * 2;
  static constexpr int NS = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + NS * kKVBytes;
  static constexpr int kOffBar = kOffV + NS * kKVBytes;
  // q_full, k_full[NS], v_full[NS], k_empty[NS], v_empty[NS], s_full[2],
  // p_half[2], p_ready[2], o_final, mask_full[kMaskRing], mask_empty[kMaskRing]
  static constexpr int kNumBars = 1 + 4 * NS + 2 + 2 + 2 + 1 + 2 * kMaskRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffTiles = kOffMisc + 16;
  static constexpr int kOffSets = kOffTiles + kMaxRuns * 12;  // run table: tok0, len, v0
  static constexpr int kOffMasks = kOffSets + (kMaxRowFrames + 1) * kSetWords * 4;
  // [kMaskRing][kMaxRowFrames] 128-bit key masks: tile j, query frame tf + slot
  static constexpr int kBytes = kOffMasks + kMaskRing * kMaxRowFrames * 16;
  static constexpr int kSmem = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct LvsaParams {
  int B, Hh, T, P, N, C, T_per, s_mod;  // T_per = 0: no anchors
  int alternate;                        // alternating window growth
  int pack;                             // runs start on 8-row (1) or 128-row (0) boundaries
  FastDiv divP;
  float scale, scale_log2;
  __nv_bfloat16* o;  // natural layout
  float* lse;        // [B, Hh, N] or null
  unsigned int* status;
  uint64_t wait_limit_ns;
};

// Maps of the same tensors with boxes of 64, 32, 16 and 8 tokens (index 3..0):
// the pieces of packed key tiles.
struct RunMaps {
  CUtensorMap k[4], v[4];
};

__device__ __forceinline__ int floordiv(int a, int b) {
  int q = a / b;
  if ((a % b != 0) && (a < 0)) --q;  // b > 0
  return q;
}

// anchors in [a, b] (frames f with f = s_mod mod T_per; none when T_per = 0)
__device__ __forceinline__ int anchors_in(int a, int b, int s_mod, int T_per) {
  return (b < a || T_per == 0) ? 0
                               : floordiv(b - s_mod, T_per) - floordiv(a - 1 - s_mod, T_per);
}

__device__ __forceinline__ bool is_anchor(int f, int s_mod, int T_per) {
  if (T_per == 0) return false;
  int r = (f - s_mod) % T_per;
  if (r < 0) r += T_per;
  return r == 0;
}

// f in A(t)?
__device__ bool lvsa_member(int t, int f, const LvsaParams& p) {
  const bool t_anchor = is_anchor(t, p.s_mod, p.T_per);
  if (f == t || is_anchor(f, p.s_mod, p.T_per)) return true;
  const int base = anchors_in(0, p.T - 1, p.s_mod, p.T_per) + (t_anchor ? 0 : 1);
  const int need = p.C - base;
  if (p.alternate) {
    // right and left pointers take turns (right first): the right side takes
    // kR of its nR frames outside the base, nearest first, the left the rest
    const int nR = (p.T - 1 - t) - anchors_in(t + 1, p.T - 1, p.s_mod, p.T_per);
    const int nL = t - anchors_in(0, t - 1, p.s_mod, p.T_per);
    const int kR = min(nR, max((need + 1) / 2, need - nL)), kL = need - kR;
    if (f > t) return (f - t) - anchors_in(t + 1, f, p.s_mod, p.T_per) <= kR;
    return (t - f) - anchors_in(f, t - 1, p.s_mod, p.T_per) <= kL;
  }
  const int d = f > t ? f - t : t - f;
  // frames outside the base strictly nearer than d (t itself is in the base)
  const int lo = max(t - d + 1, 0), hi = min(t + d - 1, p.T - 1);
  int before = (hi - lo + 1) - anchors_in(lo, hi, p.s_mod, p.T_per) - (t_anchor ? 0 : 1);
  // at equal distance the right-hand frame comes first
  if (f < t && t + d < p.T && !is_anchor(t + d, p.s_mod, p.T_per)) ++before;
  return before < need;
}

__device__ __forceinline__ bool bit_of(const uint32_t* set, int f) {
  return (set[f >> 5] >> (f & 31)) & 1u;
}

// first f' >= f (f' < T) with bit value `v` in `set`, else T
__device__ int next_with(const uint32_t* set, int f, int T, bool v) {
  while (f < T) {
    uint32_t w = set[f >> 5];
    if (!v) w = ~w;
    w &= kFullMask << (f & 31);
    if (w) {
      const int g = (f & ~31) + __ffs(w) - 1;
      return g < T ? g : T;
    }
    f = (f & ~31) + 32;
  }
  return T;
}

__device__ __forceinline__ void cta_end_sync() { asm volatile("bar.sync 2, 384;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    lvsa_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const LvsaParams p,
                     const __grid_constant__ RunMaps rm) {
  using Cfg = LvsaCfg<D>;
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
  uint64_t* s_full = v_empty + Cfg::NS;   // [2]
  uint64_t* p_half = s_full + 2;          // [2]: keys 0..63 of P stored
  uint64_t* p_ready = p_half + 2;         // [2]: all of P stored
  uint64_t* o_final = p_ready + 2;
  uint64_t* mask_full = o_final + 1;            // [kMaskRing]: masks of a tile written
  uint64_t* mask_empty = mask_full + kMaskRing;  // [kMaskRing]: read by the 8 softmax warps
  uint4* masks = reinterpret_cast<uint4*>(smem + Cfg::kOffMasks);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);  // tmem, abort, ntiles, skip
  // runs of consecutive frames of the union, laid end to end as a stream of
  // key rows: run r = tokens [run_tok[r], + run_len[r]) at rows run_v[r]..
  int32_t* run_tok = reinterpret_cast<int32_t*>(smem + Cfg::kOffTiles);
  int32_t* run_len = run_tok + kMaxRuns;
  int32_t* run_v = run_len + kMaxRuns;
  uint32_t* sets = reinterpret_cast<uint32_t*>(smem + Cfg::kOffSets);  // [rf][kSetWords], union last
  uint32_t* uset = sets + kMaxRowFrames * kSetWords;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = pair * kPair;
  const int64_t brow = (int64_t)b * p.N;
  const int q_last = min(q0 + kPair, p.N) - 1;
  const int tf = (int)p.divP.div((uint32_t)q0);
  const int nrf = (int)p.divP.div((uint32_t)q_last) - tf + 1;
  const int words = (p.T + 31) >> 5;
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
    for (int i = 0; i < kMaskRing; ++i) {
      mbar_init(&mask_full[i], 32);
      mbar_init(&mask_empty[i], 8);
    }
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = (*reinterpret_cast<volatile unsigned int*>(p.status) & kStatusTimeout) ? 1u : 0u;
    fence_mbar_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  // packed key tiles leave rows between and after their pieces: masked, but
  // P = 0 times a value must stay 0, so V stages start at zero
  if (p.pack) {
    for (int i = threadIdx.x; i < Cfg::NS * Cfg::kKVBytes / 16; i += kThreads)
      reinterpret_cast<uint4*>(smem + Cfg::kOffV)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (misc[3]) return;
  if (warp == 1) {
    tmem_alloc(&misc[0], Cfg::kTmemCols);
    tmem_relinquish();
  }
  // frame sets of the query frames tf .. tf+nrf-1 (one 32-frame word per step)
  for (int idx = threadIdx.x; idx < nrf * words; idx += kThreads) {
    const int rf = idx / words, w = idx - rf * words;
    uint32_t bits = 0u;
    for (int i = 0; i < 32; ++i) {
      const int f = 32 * w + i;
      if (f < p.T && lvsa_member(tf + rf, f, p)) bits |= 1u << i;
    }
    sets[rf * kSetWords + w] = bits;
  }
  __syncthreads();
  for (int w = threadIdx.x; w < words; w += kThreads) {
    uint32_t u = 0u;
    for (int rf = 0; rf < nrf; ++rf) u |= sets[rf * kSetWords + w];
    uset[w] = u;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the runs of consecutive frames of U, end to end: a run starts on the
    // next 8-row boundary after the previous one (the 128-byte swizzle
    // atom) when frames are a multiple of 8 tokens, so the tail of one run
    // shares its key tile with the head of the next; otherwise on the next
    // 128-row boundary.  Key tile j = stream rows [128 j, 128 j + 128).
    const int align = p.pack ? 8 : kTile;
    int nr = 0, v = 0;
    bool overflow = false;
    for (int f = next_with(uset, 0, p.T, true); f < p.T;) {
      const int e = next_with(uset, f, p.T, false);  // run [f, e)
      if (nr < kMaxRuns) {
        run_tok[nr] = f * p.P;
        run_len[nr] = (e - f) * p.P;
        run_v[nr] = v;
        v = (v + (e - f) * p.P + align - 1) / align * align;
        ++nr;
      } else {
        overflow = true;
      }
      f = next_with(uset, e, p.T, true);
    }
    if (overflow) atomicOr(p.status, kStatusBadBlocklist);
    misc[2] = (v + kTile - 1) / kTile;
    misc[3] = nr;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];
  const int n = (int)misc[2];
  const int nruns = (int)misc[3];
  // pieces of key tile j: [row offset, first token, length] of each run it
  // meets, walked with a cursor (tiles are visited in order)
  auto first_run = [&](int j, int& r) {
    while (r < nruns && run_v[r] + run_len[r] <= j * kTile) ++r;
  };

  // register split: 128 threads x 72 + 256 threads x 216 = 64512, the 384 x
  // 168 registers the block is launched with (fewer for the issuing warps
  // made them spill, and each reload delayed an MMA batch)
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
    if (warp == 2 && n > 0) {
      // ------------------------------------------------------ key masks
      // lane rf computes, for key tile j, which of its 128 rows the queries
      // of frame tf + rf attend: rows of frames in A(tf + rf); rows between
      // and after the pieces stay masked.  The softmax warps read them from
      // a ring of kMaskRing tiles.
      int rcur = 0;
      const uint32_t* myset = sets + min(lane, kMaxRowFrames - 1) * kSetWords;
      for (int j = 0; j < n; ++j) {
        const int r = j % kMaskRing;
        if (!__all_sync(kFullMask, bounded_wait(&mask_empty[r], ((j / kMaskRing) & 1) ^ 1, wc)))
          break;
        first_run(j, rcur);
        uint32_t vm[4] = {0u, 0u, 0u, 0u};
        for (int rr = rcur; rr < nruns && run_v[rr] < (j + 1) * kTile; ++rr) {
          const int a = max(j * kTile, run_v[rr]), e = min((j + 1) * kTile, run_v[rr] + run_len[rr]);
          if (e <= a) continue;
          const int k0 = run_tok[rr] + (a - run_v[rr]), kn = e - a, o = a - j * kTile;
          int f = (int)p.divP.div((uint32_t)k0);
          int lo = 0, fend = (f + 1) * p.P - k0;
          while (lo < kn) {
            const int hi = min(kn, fend);
            if (f < p.T && bit_of(myset, f)) set_range(vm, o + lo, o + hi);
            lo = hi;
            ++f;
            fend += p.P;
          }
        }
        if (lane < nrf) masks[r * kMaxRowFrames + lane] = make_uint4(vm[0], vm[1], vm[2], vm[3]);
        __syncwarp();
        mbar_arrive(&mask_full[r]);
      }
    } else if (warp == 0 && n > 0) {
      // -------------------------------------------------------- TMA producer
      // the whole warp runs the loop (warp-uniform operands); one lane issues
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
        for (int g = 0; g < 2; ++g)
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_3d(sQ + g * Cfg::kQBytes + c * Cfg::kPanel, &tmq, q_full, c * 64, h,
                        (int)(brow + q0 + g * kTile));
      }
      __syncwarp();
      int issued_k = 0, issued_v = 0;
      int rcur = 0;
      // one key tile into `dst`: a 128-token box at the tile's first token
      // (128-row runs), or each run's piece with boxes of 128/64/32/16/8
      // tokens at its row offset (packed runs, pieces of multiples of 8)
      auto load_tile = [&](int j, int r0, uint8_t* dst, uint64_t* bar, const CUtensorMap* m128,
                           const CUtensorMap* msmall) {
        if (!p.pack) {
          const int krow = (int)(brow + run_tok[r0] + (j * kTile - run_v[r0]));
          mbar_arrive_expect_tx(bar, Cfg::kKVBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_3d(dst + c * Cfg::kPanel, m128, bar, c * 64, h, krow);
          return;
        }
        uint32_t bytes = 0;
        for (int r = r0; r < nruns && run_v[r] < (j + 1) * kTile; ++r) {
          const int a = max(j * kTile, run_v[r]), e = min((j + 1) * kTile, run_v[r] + run_len[r]);
          if (e > a) bytes += (uint32_t)(e - a) * 128u * Cfg::kChunks;
        }
        mbar_arrive_expect_tx(bar, bytes);
        for (int r = r0; r < nruns && run_v[r] < (j + 1) * kTile; ++r) {
          const int a = max(j * kTile, run_v[r]), e = min((j + 1) * kTile, run_v[r] + run_len[r]);
          if (e <= a) continue;
          int tok = run_tok[r] + (a - run_v[r]), row = a - j * kTile;
          const int len8 = (e - a) >> 3;
          for (int bsz = 4; bsz >= 0; --bsz) {
            if (!((len8 >> bsz) & 1)) continue;
            const CUtensorMap* m = bsz == 4 ? m128 : &msmall[bsz];
            for (int c = 0; c < Cfg::kChunks; ++c)
              tma_load_3d(dst + c * Cfg::kPanel + row * 128, m, bar, c * 64, h, (int)(brow + tok));
            tok += 8 << bsz;
            row += 8 << bsz;
          }
        }
      };
      for (int j = 0; j < n; ++j) {
        const int st = j % Cfg::NS;
        const uint32_t par = ((j / Cfg::NS) & 1) ^ 1;
        first_run(j, rcur);
        if (!__all_sync(kFullMask, bounded_wait(&k_empty[st], par, wc))) break;
        if (elect_one())
          load_tile(j, rcur, smem + Cfg::kOffK + st * Cfg::kKVBytes, &k_full[st], &tmk, rm.k);
        __syncwarp();
        issued_k = j + 1;
        if (!__all_sync(kFullMask, bounded_wait(&v_empty[st], par, wc))) break;
        if (elect_one())
          load_tile(j, rcur, smem + Cfg::kOffV + st * Cfg::kKVBytes, &v_full[st], &tmv, rm.v);
        __syncwarp();
        issued_v = j + 1;
      }
      if (*wc.abort) {
        // leave no copy in flight: wait (bounded, ignoring the abort flag)
        // for the loads still owned by the rings
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
      // the whole warp runs the loop (descriptors stay warp-uniform); the
      // elected lane issues the tcgen05 instructions
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
      // shared-memory descriptors: constant high word, 32-bit low words
      constexpr uint32_t dhi = sdesc_sw128_hi(1024);
      const uint32_t q_lo = sdesc_sw128_lo(smem_u32(sQ), 16);
      const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + Cfg::kOffK), 16);
      const uint32_t v_lo = sdesc_sw128_lo(smem_u32(smem + Cfg::kOffV), Cfg::kPanel);
      auto issue_qk = [&](int g, int st) {
        const uint32_t dst = tbase + g * 128;
        const uint32_t qd = q_lo + ((g * Cfg::kQBytes) >> 4);
        const uint32_t kd = k_lo + ((st * Cfg::kKVBytes) >> 4);
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
      // O_g += P(keys 64 * half .. + 63) . V(same keys)
      auto issue_pv = [&](int g, int st, int half, uint32_t acc) {
        const uint32_t dst = tbase + 256 + g * 128, pa = tbase + g * 128 + 64 + half * 32;
        const uint32_t vd = v_lo + ((st * Cfg::kKVBytes + half * 8192) >> 4);
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
    cta_end_sync();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tbase, Cfg::kTmemCols);
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
    const int qn = q0 + g * kTile + row;  // query token within the batch
    const bool qvalid = qn < p.N;
    const int tq = qvalid ? (int)p.divP.div((uint32_t)qn) : 0;
    const float sl2 = p.scale_log2;
    const float thr = 8.0f / sl2;
    RowState st;
    bool alive = true;
    const int slot = qvalid ? tq - tf : 0;
    for (int j = 0; j < n; ++j) {
      // keys of tile j allowed for this row (those whose frame is in A(tq)),
      // from the mask warp
      const int r = j % kMaskRing;
      if (!__all_sync(kFullMask, bounded_wait(&mask_full[r], (j / kMaskRing) & 1, wc))) {
        alive = false;
        break;
      }
      const uint4 mv = masks[r * kMaxRowFrames + slot];
      const uint32_t vm[4] = {qvalid ? mv.x : 0u, qvalid ? mv.y : 0u, qvalid ? mv.z : 0u,
                              qvalid ? mv.w : 0u};
      __syncwarp();
      if (lane == 0) mbar_arrive(&mask_empty[r]);
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
      // S of tile j was written after PV of tile j-1: O is complete here
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
    const bool has = alive && n > 0 && qvalid && st.l > 0.f;
    const float inv_l = has ? 1.f / st.l : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(p.o + ((brow + qn) * p.Hh + h) * D);
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
        w16[i] = pack_bf16x2(__uint_as_float(o32[2 * i]) * inv_l,
                             __uint_as_float(o32[2 * i + 1]) * inv_l);
      if (qvalid) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[c * 4 + i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
      }
    }
    if (qvalid && p.lse)
      p.lse[((int64_t)b * p.Hh + h) * p.N + qn] = has ? st.m * p.scale + logf(st.l) : -INFINITY;
    tc_fence_before();
    cta_end_sync();
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn3() {
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

// Natural layout [B*N, Hh, D] bf16: boxes of 64 channels x 1 head x `rows`
// tokens.
bool make_tmap_natural(CUtensorMap* m, const void* ptr, int64_t tokens, int Hh, int D,
                       int rows = kTile) {
  auto fn = encode_fn3();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hh, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hh * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_lvsa_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const LvsaParams& p, const RunMaps& rm, dim3 grid, cudaStream_t st) {
  auto kern = lvsa_attn_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LvsaCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, LvsaCfg<D>::kSmem, st>>>(q, k, v, p, rm);
  return cudaGetLastError();
}

}  // namespace

}  // namespace bsa

using namespace bsa;

extern "C" bsa_status bsa_lvsa_attn_fwd(bsa_plan_t plan, int C, int T_per, int s, const void* q,
                                        const void* k, const void* v, float scale, void* o,
                                        float* lse, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_FRAME) return set_error(BSA_ERR_INVALID_ARG, "LVSA attention needs a FRAME plan");
  if (T_per < 1) return set_error(BSA_ERR_INVALID_ARG, "T_per must be >= 1");
  if (C < 1 || C > g.T) return set_error(BSA_ERR_INVALID_ARG, "C must be in [1, T]");
  if (!(scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be positive");
  for (const void* ptr : {q, k, v, (const void*)o}) {
    if (!ptr) return set_error(BSA_ERR_INVALID_ARG, "q / k / v / o is NULL");
    if (!aligned16(ptr)) return set_error(BSA_ERR_ALIGNMENT, "q / k / v / o not 16-byte aligned");
  }
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "lse is not 4-byte aligned");
  int tp = 0, sm = 0;
  const int anchors = lvsa_effective_anchors(plan, T_per, s, &tp, &sm);
  if (anchors + (anchors < g.T ? 1 : 0) > C)
    return set_error(BSA_ERR_INVALID_ARG, "budget C is smaller than the anchors plus the query frame");
  if (g.T > kMaxFrames) return set_error(BSA_ERR_UNSUPPORTED, "fused LVSA attention supports T <= 4096");
  if (g.P < 37) return set_error(BSA_ERR_UNSUPPORTED, "fused LVSA attention needs >= 37 tokens per frame");
  const int64_t N = (int64_t)g.T * g.P;
  if ((int64_t)g.B * N >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (N >= (1 << 24)) return set_error(BSA_ERR_UNSUPPORTED, "fused LVSA attention needs N < 2^24");
  // runs of a query pair's union: at most |U| <= min(T, rows' frames * C)
  const int64_t u_frames = std::min<int64_t>(g.T, (int64_t)kMaxRowFrames * C);
  if (u_frames > kMaxRuns)
    return set_error(BSA_ERR_UNSUPPORTED, "fused LVSA attention: too many frames per query pair");
  CUtensorMap tq, tk, tv;
  const int64_t tokens = (int64_t)g.B * N;
  if (!make_tmap_natural(&tq, q, tokens, g.Hh, g.D) || !make_tmap_natural(&tk, k, tokens, g.Hh, g.D) ||
      !make_tmap_natural(&tv, v, tokens, g.Hh, g.D))
    return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  LvsaParams p;
  p.B = g.B;
  p.Hh = g.Hh;
  p.T = g.T;
  p.P = g.P;
  p.N = (int)N;
  p.C = C;
  p.T_per = tp;
  p.s_mod = sm;
  p.alternate = plan->lvsa_window == BSA_WINDOW_ALTERNATE ? 1 : 0;
  p.pack = (g.P % 8 == 0) ? 1 : 0;
  RunMaps rm;
  memset(&rm, 0, sizeof(rm));
  if (p.pack)
    for (int b = 0; b < 4; ++b)
      if (!make_tmap_natural(&rm.k[b], k, tokens, g.Hh, g.D, 8 << b) ||
          !make_tmap_natural(&rm.v[b], v, tokens, g.Hh, g.D, 8 << b))
        return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D, small boxes) failed");
  p.divP = FastDiv((uint32_t)g.P);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = plan->d_status;
  p.wait_limit_ns = plan->wait_limit_ns;
  const dim3 grid((unsigned)((N + kPair - 1) / kPair), (unsigned)g.Hh, (unsigned)g.B);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = g.D == 128 ? launch_lvsa_t<128>(tq, tk, tv, p, rm, grid, st)
                                   : launch_lvsa_t<64>(tq, tk, tv, p, rm, grid, st);
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "lvsa_attn launch");
}

