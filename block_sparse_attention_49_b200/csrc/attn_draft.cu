// Draft attention on the natural layout, persistent: one CTA per SM walks
// its share of the query tiles and keeps its pipelines running across them.
//
// What it computes (Draft Attention article: the sparse mask from the draft
// map guides full-resolution block-sparse attention; the reorder that makes
// the kept blocks contiguous is fused into the tile loads and stores): for
// every query token, softmax(scale * q.k) over the tokens of the key tiles
// its query tile keeps, weighted sum of their values; the same result as
// bsa_attn_fwd on reordered tensors followed by the inverse reorder.
//
// Why persistent: a draft row keeps a few dozen key tiles (34 of 336 at 90 %
// sparsity), so a CTA per query tile spends a share of its life on set-up
// and on loads that no earlier work hides.  Here the next tile's list,
// query tile and first key tiles load while the current tile finishes.
// Measured on the Wan-14B-like draft workload (keep 4 to 34 blocks per
// row): 0.67 ms + 0.080 ms per kept block, against 0.74 ms + 0.078 ms with
// a CTA per query tile.  The remaining per-tile cost is the tile's own
// ramp: its first softmax waits for its first QK, and its epilogue (the
// two groups' merge and the stores) runs on the softmax warps before the
// next tile's softmax can start.
//
// Roles (12 warps; tile i = the i-th query tile of this CTA):
//   warp 0      TMA producer of Q (after the last QK of tile i-1) and of K
//               into a 3-deep ring; warp 3 of V into a 2-deep ring (K is
//               needed a softmax earlier than V).  Edge tiles (partial tiles
//               at the grid's right and bottom edges) are packed several to
//               a 128-row MMA tile, each piece loaded with a box of its
//               exact size.
//   warp 1      MMA issuer: S = Q K^T into the group's S buffer, O += P V;
//               the first PV of tile i waits until tile i-1's output has
//               been read out of tensor memory.
//   warp 2      scheduler: the key list of tile i, sorted by tile kind for
//               packing, into one of two list buffers.
//   warps 4-7   softmax group A (key tiles 0, 2, 4, ... of a query tile),
//   warps 8-11  group B (1, 3, 5, ...): one row per thread, running max and
//               sum, P as bf16 over its S; then the epilogue of the tile:
//               the two groups' partial results merged (a split-key
//               combine), normalised and stored to the tokens.
// Tensor memory: S_A | S_B | O_A | O_B (512 columns).  The arithmetic per
// tile is that of bsa_attn_fwd, so on a grid without partial tiles the
// result is identical, bit for bit, to the reorder path.
// Every wait is bounded; a wait that runs out records a timeout in the
// plan's status word and the CTA leaves without trapping.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 384;
constexpr int kListMax = 768;           // key-list entries a tile can pack
constexpr uint16_t kBad = 0xffffu;      // packed-list marker of an out-of-range entry
constexpr uint32_t kAll = 0xffffffffu;

template <int D>
struct DraftCfg {
  static constexpr int kChunks = D / 64;          // 128-byte swizzle panels
  static constexpr int kPanel = kTile * 128;
  static constexpr int kTileBytes = kTile * D * 2;
  // K and V have rings of their own: K is needed a softmax earlier than V
  // (QK of the next tile is issued before PV of this one), so it runs deeper
  static constexpr int NK = 3, NV = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTileBytes;
  static constexpr int kOffV = kOffK + NK * kTileBytes;
  static constexpr int kOffBar = kOffV + NV * kTileBytes;
  // q_full, q_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  // s_full[2], p_ready[2], o_final, o_free, list_full[2], list_empty[2]
  static constexpr int kNumBars = 2 + 2 * NK + 2 * NV + 2 + 2 + 2 + 2 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;     // tmem, abort
  static constexpr int kOffStats = kOffMisc + 16;             // [4][128] floats
  static constexpr int kOffLists = kOffStats + 4 * kTile * 4;
  static constexpr int kListBytes = kListMax * 2 + 32;        // entries + header
  static constexpr int kBytes = kOffLists + 2 * kListBytes;
  static constexpr int kSmem = kBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Header of a list buffer (after the entries).
struct ListHead {
  int64_t rs;    // first entry in col_idx
  int n;         // key tiles to run (packed count, or the raw length)
  int packed;    // 1: entries sorted by kind in this buffer
  int nF;        // full tiles first, then the edge pieces
  int c[3];      // edge pieces per kind (in decreasing size)
};

struct DraftParams {
  int B, Hh, T, H, W, N, TW, TH, ph, pw;
  int64_t nblocks, ntiles, total_tiles;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int per_head;
  int64_t nlists;
  float scale, scale_log2;
  __nv_bfloat16* o;
  float* lse;
  const uint32_t* tile_valid;
  unsigned int* status;
  uint64_t wait_limit_ns;
  FastDiv div_tile_frame, div_TW, div_pw;
  int pk_on;
  int pk_kind[3], pk_rows[3], pk_step[3];
};

struct DraftEdgeMaps {
  CUtensorMap k[3], v[3];
};

__device__ __forceinline__ void set_rows(uint32_t (&m)[4], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int a = max(lo, 32 * w), e = min(hi, 32 * w + 32);
    if (e > a) m[w] |= (e - a == 32 ? kAll : ((1u << (e - a)) - 1u)) << (a - 32 * w);
  }
}

// Next packed tile of edge pieces: as many of each kind as fit in 128 rows,
// largest kind first; r[] = pieces left.
__device__ __forceinline__ void next_bin(const DraftParams& p, int (&r)[3], int (&a)[3]) {
  int cap = kTile;
#pragma unroll
  for (int e = 0; e < 3; ++e) {
    a[e] = p.pk_step[e] > 0 ? min(r[e], cap / p.pk_step[e]) : 0;
    cap -= a[e] * p.pk_step[e];
    r[e] -= a[e];
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2_d(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void end_sync() { asm volatile("bar.sync 2, 384;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_draft_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DraftParams p,
                      const __grid_constant__ DraftEdgeMaps em) {
  using Cfg = DraftCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + Cfg::NK;
  uint64_t* v_full = k_empty + Cfg::NK;
  uint64_t* v_empty = v_full + Cfg::NV;
  uint64_t* s_full = v_empty + Cfg::NV;   // [2]
  uint64_t* p_ready = s_full + 2;         // [2]
  uint64_t* o_final = p_ready + 2;
  uint64_t* o_free = o_final + 1;
  uint64_t* list_full = o_free + 1;       // [2]
  uint64_t* list_empty = list_full + 2;   // [2]
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);  // tmem, abort, skip
  float* stats = reinterpret_cast<float*>(smem + Cfg::kOffStats);
  auto list_entries = [&](int buf) {
    return reinterpret_cast<uint16_t*>(smem + Cfg::kOffLists + buf * Cfg::kListBytes);
  };
  auto list_head = [&](int buf) {
    return reinterpret_cast<ListHead*>(smem + Cfg::kOffLists + buf * Cfg::kListBytes + kListMax * 2);
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{p.status, reinterpret_cast<volatile int*>(&misc[1]), p.wait_limit_ns};
  // this CTA's query tiles: u = blockIdx.x + i * gridDim.x, query tile fastest
  const int64_t my_tiles =
      p.total_tiles > blockIdx.x ? (p.total_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto tile_of = [&](int64_t i, int& qt, int& h, int& b) {
    const int64_t u = blockIdx.x + i * gridDim.x;
    qt = (int)(u % p.ntiles);
    const int64_t bh = u / p.ntiles;
    h = (int)(bh % p.Hh);
    b = (int)(bh / p.Hh);
  };
  // tile kt of (b, .) is the ph x pw tile (t, i, j): TMA coordinates
  auto nat_coords = [&](int kt, int b, int& x0, int& y0, int& fr) {
    const int t = (int)p.div_tile_frame.div((uint32_t)kt);
    const int r = kt - t * (int)p.div_tile_frame.d;
    const int i = (int)p.div_TW.div((uint32_t)r);
    x0 = (r - i * p.TW) * p.pw;
    y0 = i * p.ph;
    fr = b * p.T + t;
  };

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < Cfg::NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < Cfg::NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_ready[0], 128);
    mbar_init(&p_ready[1], 128);
    mbar_init(o_final, 1);
    mbar_init(o_free, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&list_full[i], 32);
      mbar_init(&list_empty[i], 2 + 1 + 256);  // producers, MMA warp, softmax threads
    }
    misc[1] = 0;
    misc[2] = (*reinterpret_cast<volatile unsigned int*>(p.status) & kStatusTimeout) ? 1u : 0u;
    fence_mbar_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  // packed tiles leave rows between and after their pieces: those rows are
  // masked, but P = 0 times a value must stay 0, so V stages start at zero
  for (int i = threadIdx.x; i < Cfg::NV * Cfg::kTileBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + Cfg::kOffV)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (misc[2] || my_tiles == 0) return;
  if (warp == 1) {
    tmem_alloc(&misc[0], 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
    if (warp == 2) {
      // ------------------------------------------------------ scheduler
      const int TT = (int)p.div_tile_frame.d;
      auto kind_of = [&](int c) {
        const int rr = c % TT, i = rr / p.TW, jj = rr - i * p.TW;
        const int right = (jj == p.TW - 1 && p.W - jj * p.pw < p.pw) ? 1 : 0;
        const int bottom = (i == p.TH - 1 && p.H - i * p.ph < p.ph) ? 2 : 0;
        return right | bottom;
      };
      for (int64_t i = 0; i < my_tiles; ++i) {
        const int buf = (int)(i & 1);
        if (!__all_sync(kAll, bounded_wait(&list_empty[buf], (uint32_t)((i >> 1) & 1) ^ 1u, wc))) break;
        int qt, h, b;
        tile_of(i, qt, h, b);
        const int64_t list = p.per_head ? (int64_t)b * p.Hh + h : 0;
        const int64_t r = list * p.nblocks + qt;
        const int64_t nnz = p.row_ptr[p.nlists * p.nblocks];
        int64_t rs = p.row_ptr[r];
        const int64_t re = p.row_ptr[r + 1];
        int n = 0;
        if (re < rs || rs < 0 || re > nnz) {
          if (lane == 0) atomicOr(p.status, kStatusBadBlocklist);
          rs = 0;
        } else {
          n = (int)(re - rs);
        }
        ListHead* hd = list_head(buf);
        uint16_t* ent = list_entries(buf);
        const bool packed = p.pk_on && n > 0 && n <= kListMax;
        int cF = 0, ce[3] = {0, 0, 0};
        if (packed) {
          // counting sort by kind: full tiles first (list order), then the
          // edge kinds in decreasing size
          for (int base = 0; base < n; base += 32) {
            const int e = base + lane;
            int kind = -1;
            if (e < n) {
              const int c = __ldg(p.col_idx + rs + e);
              kind = (c >= 0 && (int64_t)c < p.nblocks) ? kind_of(c) : 0;
            }
            cF += __popc(__ballot_sync(kAll, kind == 0));
#pragma unroll
            for (int k = 0; k < 3; ++k)
              ce[k] += __popc(__ballot_sync(kAll, kind > 0 && kind == p.pk_kind[k]));
          }
          int wF = 0, we[3] = {0, 0, 0};
          const int start[3] = {cF, cF + ce[0], cF + ce[0] + ce[1]};
          const uint32_t lt = (1u << lane) - 1u;
          bool bad = false;
          for (int base = 0; base < n; base += 32) {
            const int e = base + lane;
            int kind = -1;
            uint16_t val = 0;
            if (e < n) {
              const int c = __ldg(p.col_idx + rs + e);
              const bool ok = c >= 0 && (int64_t)c < p.nblocks;
              bad |= !ok;
              kind = ok ? kind_of(c) : 0;
              val = ok ? (uint16_t)c : kBad;
            }
            const uint32_t bF = __ballot_sync(kAll, kind == 0);
            int pos = kind == 0 ? wF + __popc(bF & lt) : 0;
            wF += __popc(bF);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
              const uint32_t bk = __ballot_sync(kAll, kind > 0 && kind == p.pk_kind[k]);
              if (kind > 0 && kind == p.pk_kind[k]) pos = start[k] + we[k] + __popc(bk & lt);
              we[k] += __popc(bk);
            }
            if (e < n) ent[pos] = val;
          }
          if (__any_sync(kAll, bad) && lane == 0) atomicOr(p.status, kStatusBadBlocklist);
        }
        int npk = n;
        if (packed) {
          int rr[3] = {ce[0], ce[1], ce[2]}, a[3];
          int nb = 0;
          while (rr[0] + rr[1] + rr[2] > 0) {
            next_bin(p, rr, a);
            ++nb;
          }
          npk = cF + nb;
        }
        if (lane == 0) {
          hd->rs = rs;
          hd->n = npk;
          hd->packed = packed ? 1 : 0;
          hd->nF = cF;
          hd->c[0] = ce[0];
          hd->c[1] = ce[1];
          hd->c[2] = ce[2];
        }
        __syncwarp();
        mbar_arrive(&list_full[buf]);  // every lane: each releases its own writes
      }
    } else if (warp == 0 || warp == 3) {
      // ------------------------------------------- TMA producers: K (+ Q), V
      const bool isK = warp == 0;
      const int NR = isK ? Cfg::NK : Cfg::NV;
      uint64_t* full = isK ? k_full : v_full;
      uint64_t* empty = isK ? k_empty : v_empty;
      const CUtensorMap* tmx = isK ? &tmk : &tmv;
      const int ring_off = isK ? Cfg::kOffK : Cfg::kOffV;
      int64_t jj = 0;           // tiles issued into this ring so far
      int64_t issued_q = 0;
      bool aborted = false;
      for (int64_t i = 0; i < my_tiles && !aborted; ++i) {
        const int buf = (int)(i & 1);
        if (!__all_sync(kAll, bounded_wait(&list_full[buf], (uint32_t)((i >> 1) & 1), wc))) break;
        const ListHead hd = *list_head(buf);
        const uint16_t* ent = list_entries(buf);
        int qt, h, b;
        tile_of(i, qt, h, b);
        if (isK) {
          // Q of this tile once the last QK of the previous one has completed
          if (!__all_sync(kAll, bounded_wait(q_empty, (uint32_t)(i & 1) ^ 1u, wc))) break;
          if (elect_one()) {
            int x0, y0, fr;
            nat_coords(qt, b, x0, y0, fr);
            mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
            for (int c = 0; c < Cfg::kChunks; ++c)
              tma_load_5d(sQ + c * Cfg::kPanel, &tmq, q_full, c * 64, h, x0, y0, fr);
          }
          __syncwarp();
          issued_q = i + 1;
        }
        int prem[3] = {hd.c[0], hd.c[1], hd.c[2]};
        const int pstart[3] = {hd.nF, hd.nF + hd.c[0], hd.nF + hd.c[0] + hd.c[1]};
        int pptr[3] = {0, 0, 0};
        for (int j = 0; j < hd.n; ++j, ++jj) {
          const int st = (int)(jj % NR);
          const uint32_t ph = (uint32_t)((jj / NR) & 1);
          if (!__all_sync(kAll, bounded_wait(&empty[st], ph ^ 1u, wc))) {
            aborted = true;
            break;
          }
          uint8_t* dst = smem + ring_off + st * Cfg::kTileBytes;
          if (hd.packed && j >= hd.nF) {
            int a[3];
            next_bin(p, prem, a);
            if (elect_one()) {
              uint32_t bytes = 0;
#pragma unroll
              for (int e = 0; e < 3; ++e) bytes += a[e] * p.pk_rows[e] * 128 * Cfg::kChunks;
              mbar_arrive_expect_tx(&full[st], bytes);
              int off = 0;
#pragma unroll
              for (int e = 0; e < 3; ++e) {
                for (int m = 0; m < a[e]; ++m) {
                  int x0, y0, fr;
                  nat_coords(ent[pstart[e] + pptr[e] + m], b, x0, y0, fr);
                  const CUtensorMap* mx = isK ? &em.k[p.pk_kind[e] - 1] : &em.v[p.pk_kind[e] - 1];
                  for (int c = 0; c < Cfg::kChunks; ++c)
                    tma_load_5d(dst + c * Cfg::kPanel + off * 128, mx, &full[st], c * 64, h, x0, y0,
                                fr);
                  off += p.pk_step[e];
                }
              }
            }
#pragma unroll
            for (int e = 0; e < 3; ++e) pptr[e] += a[e];
          } else {
            int kt;
            if (hd.packed) {
              const uint16_t c = ent[j];
              kt = c == kBad ? 0 : c;
            } else {
              const int c = __ldg(p.col_idx + hd.rs + j);
              const bool ok = c >= 0 && (int64_t)c < p.nblocks;
              if (!ok && isK && lane == 0) atomicOr(p.status, kStatusBadBlocklist);
              kt = ok ? c : 0;
            }
            if (elect_one()) {
              int x0, y0, fr;
              nat_coords(kt, b, x0, y0, fr);
              mbar_arrive_expect_tx(&full[st], Cfg::kTileBytes);
              for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_5d(dst + c * Cfg::kPanel, tmx, &full[st], c * 64, h, x0, y0, fr);
            }
          }
          __syncwarp();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&list_empty[buf]);
      }
      if (*wc.abort) {
        // leave no copy in flight: wait (bounded, ignoring the abort flag)
        // for the loads still owned by the ring (and the last Q)
        volatile int no_abort = 0;
        const WaitCtx drain{p.status, &no_abort, p.wait_limit_ns};
        if (isK && issued_q > 0) bounded_wait(q_full, (uint32_t)((issued_q - 1) & 1), drain);
        for (int64_t q = std::max<int64_t>(0, jj - NR); q < jj; ++q)
          bounded_wait(&full[q % NR], (uint32_t)((q / NR) & 1), drain);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
      const uint64_t qd = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t vd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffV), Cfg::kPanel, 1024);
      auto issue_qk = [&](int st, uint32_t tdst) {
        const uint64_t kd = sdesc_add(kd0, st * Cfg::kTileBytes);  // K ring stage
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * Cfg::kPanel + (kk & 3) * 32;
            mma_ss(tdst, sdesc_add(qd, off), sdesc_add(kd, off), idesc_qk, kk > 0);
          }
        }
        __syncwarp();
      };
      auto issue_pv = [&](int st, uint32_t tP, uint32_t tO, uint32_t acc) {
        const uint64_t vd = sdesc_add(vd0, st * Cfg::kTileBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tO, tP + kk * 8, sdesc_add(vd, kk * 16 * 128), idesc_pv, (acc | (uint32_t)kk) != 0);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) mma_commit(bar);
        __syncwarp();
      };
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(kAll, bounded_wait(bar, parity, wc));
      };
      int64_t jj = 0;             // key tiles consumed so far (ring position)
      int64_t pcount[2] = {0, 0};  // completed P hand-offs per group
      bool alive = true;
      for (int64_t i = 0; alive && i < my_tiles; ++i) {
        const int buf = (int)(i & 1);
        if (!wait(&list_full[buf], (uint32_t)((i >> 1) & 1))) break;
        const int n = list_head(buf)->n;
        __syncwarp();
        if (lane == 0) mbar_arrive(&list_empty[buf]);
        if (!wait(q_full, (uint32_t)(i & 1))) break;
        tc_fence_after();
        if (n > 0) {
          const int st0 = (int)(jj % Cfg::NK);
          if (!wait(&k_full[st0], (uint32_t)((jj / Cfg::NK) & 1))) break;
          tc_fence_after();
          issue_qk(st0, tbase);
          commit(&s_full[0]);
          commit(&k_empty[st0]);
        }
        if (n <= 1) commit(q_empty);  // Q no longer read once that QK completes
        for (int j = 0; j < n; ++j) {
          if (j + 1 < n) {
            const int64_t q1 = jj + j + 1;
            const int st1 = (int)(q1 % Cfg::NK);
            if (!wait(&k_full[st1], (uint32_t)((q1 / Cfg::NK) & 1))) { alive = false; break; }
            tc_fence_after();
            issue_qk(st1, tbase + ((j + 1) & 1) * 128);
            commit(&s_full[(j + 1) & 1]);
            commit(&k_empty[st1]);
            if (j + 2 == n) commit(q_empty);
          }
          const int g = j & 1;
          const int64_t q0 = jj + j;
          const int st = (int)(q0 % Cfg::NV);
          if (!wait(&p_ready[g], (uint32_t)(pcount[g] & 1)) ||
              !wait(&v_full[st], (uint32_t)((q0 / Cfg::NV) & 1))) {
            alive = false;
            break;
          }
          ++pcount[g];
          // the previous tile's output must be out of tensor memory before
          // this tile's first PV overwrites O
          if (j == 0 && i > 0 && !wait(o_free, (uint32_t)((i - 1) & 1))) { alive = false; break; }
          tc_fence_after();
          issue_pv(st, tbase + g * 128 + 64, tbase + 256 + g * 128, j >= 2);
          commit(&v_empty[st]);
        }
        jj += n;
        if (n == 0 && i > 0 && !wait(o_free, (uint32_t)((i - 1) & 1))) alive = false;
        commit(o_final);
      }
    }
    end_sync();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tbase, 512);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    // -------------------------------------------------------- softmax groups
    const int g = (warp >= 8) ? 1 : 0;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + g * 128 + lane_off;
    const uint32_t tO = tbase + 256 + g * 128 + lane_off;
    const float sl2 = p.scale_log2;
    const float thr = 8.0f / sl2;  // rescale O when the max grows by more than 2^8
    int64_t scount = 0;            // S buffers of this group consumed so far
    bool alive = true;
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int buf = (int)(i & 1);
      if (!__all_sync(kAll, bounded_wait(&list_full[buf], (uint32_t)((i >> 1) & 1), wc))) {
        alive = false;
        break;
      }
      const ListHead hd = *list_head(buf);
      const uint16_t* ent = list_entries(buf);
      int qt, h, b;
      tile_of(i, qt, h, b);
      const int n = hd.n;
      float m_run = -INFINITY, l_run = 0.f;
      int srem[3] = {hd.c[0], hd.c[1], hd.c[2]};
      int scur = hd.nF;
      for (int j = g; j < n; j += 2) {
        uint32_t vm[4] = {0u, 0u, 0u, 0u};
        if (hd.packed && j >= hd.nF) {
          int a[3];
          while (scur < j) {
            next_bin(p, srem, a);
            ++scur;
          }
          next_bin(p, srem, a);
          ++scur;
          int off = 0;
#pragma unroll
          for (int e = 0; e < 3; ++e)
            for (int m = 0; m < a[e]; ++m) {
              set_rows(vm, off, off + p.pk_rows[e]);
              off += p.pk_step[e];
            }
        } else {
          int kt;
          bool ok;
          if (hd.packed) {
            const uint16_t c = ent[j];
            ok = c != kBad;
            kt = ok ? c : 0;
          } else {
            const int c = __ldg(p.col_idx + hd.rs + j);
            ok = c >= 0 && (int64_t)c < p.nblocks;
            kt = ok ? c : 0;
          }
          const uint4 tv = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + kt);
          vm[0] = ok ? tv.x : 0u;
          vm[1] = ok ? tv.y : 0u;
          vm[2] = ok ? tv.z : 0u;
          vm[3] = ok ? tv.w : 0u;
        }
        if (!__all_sync(kAll, bounded_wait(&s_full[g], (uint32_t)(scount & 1), wc))) {
          alive = false;
          break;
        }
        ++scount;
        tc_fence_after();
        float s[128];
        {
          uint32_t r128[128];
          tmem_ld128(tS, r128);
#pragma unroll
          for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(r128[e]);
        }
        if ((vm[0] & vm[1] & vm[2] & vm[3]) != kAll) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (!((vm[w] >> e) & 1u)) s[w * 32 + e] = -INFINITY;
        }
        // row max: 8 independent chains of 3-input max, then a small tree
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmax3f(s[c], s[c + 8], s[c + 16]);
#pragma unroll
        for (int e = 24; e < 120; e += 16)
#pragma unroll
          for (int c = 0; c < 8; ++c) m8[c] = fmax3f(m8[c], s[e + c], s[e + 8 + c]);
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(m8[c], s[120 + c]);
        const float mx = fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]),
                                fmaxf(m8[6], m8[7]));
        const float m_new = fmaxf(m_run, mx);
        const bool need = m_new > m_run + thr;
        float corr = 1.f;
        if (need) {
          corr = ex2_approx((m_run - m_new) * sl2);
          m_run = m_new;
          l_run *= corr;
        }
        const float ms = (m_run == -INFINITY) ? 0.f : m_run * sl2;
        uint32_t pk[64];
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float p0 = ex2_approx(fmaf(s[2 * e], sl2, -ms));
          const float p1 = ex2_approx(fmaf(s[2 * e + 1], sl2, -ms));
          l8[e & 7] += p0 + p1;
          pk[e] = pack_bf16x2_d(p0, p1);
        }
        l_run += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        // O of this group holds every earlier PV of the group in this tile:
        // S(j) was written after the group's previous PV
        if (j >= 2 && __any_sync(kAll, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o32[32];
            tmem_ld32(tO + c * 32, o32);
#pragma unroll
            for (int e = 0; e < 32; ++e) o32[e] = __float_as_uint(__uint_as_float(o32[e]) * corr);
            tmem_st32(tO + c * 32, o32);
          }
        }
        tmem_st32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tc_fence_before();
        mbar_arrive(&p_ready[g]);
      }
      mbar_arrive(&list_empty[buf]);
      if (!alive) break;
      // ------------------------------------------------------ epilogue
      if (!__all_sync(kAll, bounded_wait(o_final, (uint32_t)(i & 1), wc))) {
        alive = false;
        break;
      }
      tc_fence_after();
      stats[(2 * g) * kTile + row] = m_run;
      stats[(2 * g + 1) * kTile + row] = l_run;
      softmax_sync();
      const float mA = stats[row], lA = stats[kTile + row];
      const float mB = stats[2 * kTile + row], lB = stats[3 * kTile + row];
      softmax_sync();  // the statistics are read before the next tile rewrites them
      const int nA = (n + 1) / 2, nB = n / 2;
      const float m = fmaxf(mA, mB);
      const float a = (nA > 0 && mA != -INFINITY) ? ex2_approx((mA - m) * sl2) : 0.f;
      const float bb = (nB > 0 && mB != -INFINITY) ? ex2_approx((mB - m) * sl2) : 0.f;
      const float l = lA * a + lB * bb;
      const uint4 tq = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + qt);
      const uint32_t qw = (row < 32) ? tq.x : (row < 64) ? tq.y : (row < 96) ? tq.z : tq.w;
      const bool qvalid = (qw >> (row & 31)) & 1u;
      const bool has = n > 0 && qvalid && l > 0.f;
      const float inv_l = has ? 1.f / l : 0.f;
      const float wa = a * inv_l, wb = bb * inv_l;
      // slot (y, x) of tile (t, i, j) is token (t, y0 + y, x0 + x)
      int x0, y0, fr;
      nat_coords(qt, b, x0, y0, fr);
      const int ay = (int)p.div_pw.div((uint32_t)row);
      const int yy = y0 + ay, xx = x0 + (row - ay * p.pw);
      const int t = fr - b * p.T;
      const int64_t ntok = ((int64_t)t * p.H + yy) * p.W + xx;
      const int64_t orow = ((int64_t)b * p.N + ntok) * p.Hh + h;
      const int64_t lrow = ((int64_t)b * p.Hh + h) * p.N + ntok;
      // group g stores columns [g*D/2, (g+1)*D/2) of its rows
      uint4* dst = reinterpret_cast<uint4*>(p.o + orow * D + g * (D / 2));
      const uint32_t oA = tbase + 256 + lane_off + g * (D / 2);
      const uint32_t oB = tbase + 384 + lane_off + g * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t xa[32], xb[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) xa[e] = xb[e] = 0u;
        if (nA > 0) tmem_ld32(oA + c * 32, xa);
        if (nB > 0) tmem_ld32(oB + c * 32, xb);
        uint32_t w16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float v0 = has ? __uint_as_float(xa[2 * e]) * wa + __uint_as_float(xb[2 * e]) * wb : 0.f;
          const float v1 =
              has ? __uint_as_float(xa[2 * e + 1]) * wa + __uint_as_float(xb[2 * e + 1]) * wb : 0.f;
          w16[e] = pack_bf16x2_d(v0, v1);
        }
        if (qvalid) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[c * 4 + e] = make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
        }
      }
      if (g == 0 && p.lse && qvalid) p.lse[lrow] = has ? m * p.scale + logf(l) : -INFINITY;
      tc_fence_before();
      mbar_arrive(o_free);
    }
    tc_fence_before();
    end_sync();
  }
}

PFN_cuTensorMapEncodeTiled_v12000 draft_encode_fn() {
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

// Natural layout [B, N, Hh, D] bf16 as 5-D {D, Hh, W, H, B*T}; boxes of 64
// channels x 1 head x box_w x box_h x 1 frame, 128-byte swizzle; boxes
// reaching past W or H read zeros.
bool make_draft_tmap(CUtensorMap* m, const void* ptr, const Geometry& g, int box_w, int box_h) {
  auto fn = draft_encode_fn();
  if (!fn) return false;
  const cuuint64_t row = (cuuint64_t)g.Hh * g.D * 2;
  cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.Hh, (cuuint64_t)g.W, (cuuint64_t)g.H,
                        (cuuint64_t)g.B * g.T};
  cuuint64_t strides[4] = {(cuuint64_t)g.D * 2, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int draft_sm_count() {
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

template <int D>
cudaError_t launch_draft_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const DraftParams& p, const DraftEdgeMaps& em, cudaStream_t st) {
  auto kern = attn_draft_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DraftCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(p.total_tiles, draft_sm_count());
  kern<<<(unsigned)grid, kThreads, DraftCfg<D>::kSmem, st>>>(q, k, v, p, em);
  return cudaGetLastError();
}

}  // namespace



bsa_status launch_attn_draft(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                             const int32_t* row_ptr, const int32_t* col_idx, int per_head,
                             float scale, void* o, float* lse, cudaStream_t st) {
  const Geometry& g = plan.g;
  if (g.layout != BSA_LAYOUT_TILE || g.block != kTile)
    return set_error(BSA_ERR_UNSUPPORTED,
                     "natural-layout attention needs a TILE plan with pool_h * pool_w = 128");
  if ((int64_t)g.B * g.T * g.P * g.Hh >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "B*N*Hh must be < 2^31");
  if ((int64_t)g.B * g.T >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "B*T must be < 2^31");
  CUtensorMap tq, tk, tv;
  if (!make_draft_tmap(&tq, q, g, g.pw, g.ph) || !make_draft_tmap(&tk, k, g, g.pw, g.ph) ||
      !make_draft_tmap(&tv, v, g, g.pw, g.ph))
    return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (5-D) failed");
  DraftParams p;
  memset(&p, 0, sizeof(p));
  p.B = g.B;
  p.Hh = g.Hh;
  p.T = g.T;
  p.H = g.H;
  p.W = g.W;
  p.N = g.T * g.P;
  p.ph = g.ph;
  p.pw = g.pw;
  p.TW = g.TW;
  p.TH = g.TH;
  p.nblocks = g.nblocks;
  p.ntiles = g.ntiles;
  p.total_tiles = (int64_t)g.B * g.Hh * g.ntiles;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.per_head = per_head ? 1 : 0;
  p.nlists = per_head ? (int64_t)g.B * g.Hh : 1;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.tile_valid = plan.d_tile_valid;
  p.status = plan.d_status;
  p.wait_limit_ns = plan.wait_limit_ns;
  p.div_tile_frame = FastDiv((uint32_t)(g.TH * g.TW));
  p.div_TW = FastDiv((uint32_t)g.TW);
  p.div_pw = FastDiv((uint32_t)g.pw);
  DraftEdgeMaps em;
  memset(&em, 0, sizeof(em));
  int kind[3] = {0, 0, 0}, rows[3] = {0, 0, 0}, bw[3] = {0, 0, 0}, bh[3] = {0, 0, 0};
  const int nk = edge_kinds(g, kind, rows, bw, bh);
  if (nk > 0 && g.nblocks < 32768) {
    for (int i = 0; i < nk; ++i) {
      p.pk_kind[i] = kind[i];
      p.pk_rows[i] = rows[i];
      p.pk_step[i] = (rows[i] + 7) / 8 * 8;
      if (!make_draft_tmap(&em.k[kind[i] - 1], k, g, bw[i], bh[i]) ||
          !make_draft_tmap(&em.v[kind[i] - 1], v, g, bw[i], bh[i]))
        return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (5-D edge boxes) failed");
    }
    p.pk_on = 1;
  }
  const cudaError_t e = g.D == 128 ? launch_draft_t<128>(tq, tk, tv, p, em, st)
                                   : launch_draft_t<64>(tq, tk, tv, p, em, st);
  if (e != cudaSuccess) return cuda_error(e, "draft attention launch");
  return BSA_OK;
}

}  // namespace bsa
