// Block-sparse attention on per-head lists of 128-slot blocks, persistent:
// one CTA per SM walks its share of the query tiles and keeps its pipelines
// running across them.  Three forms of the same body:
//   natural layout (bf16): the draft path without reorders;
//   natural layout, e4m3 tiles (template flag F8): the 8-bit draft path;
//   slot mode: [B, Hh, Npad, D] slot tensors of any plan (bsa_attn_fwd with
//   per-head lists).
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
// query tile and first key tiles load while the current tile finishes.  The
// remaining per-tile cost is the tile's own ramp: its first softmax waits
// for its first QK, and its epilogue (the two groups' merge and the stores)
// runs on the softmax warps before the next tile's softmax can start.
//
// Roles (12 warps; tile i = the i-th query tile of this CTA):
//   warp 0      TMA producer of Q (after the last QK of tile i-1) and of K
//               into a ring (3 deep, 4 for e4m3); warp 3 of V into a ring
//               (2 deep, 4 for e4m3): K is needed a softmax earlier than V.
//               On the tile layout (natural tensors, or the slots of a
//               TILE plan), edge tiles (partial tiles at the grid's right
//               and bottom edges) are packed several to a 128-row MMA
//               tile, each piece loaded with a box of its exact size.
//   warp 1      MMA issuer: a group's PV in two halves as its P halves
//               arrive, then that group's next QK; the first PV of tile i
//               waits until tile i-1's output has been read out of tensor
//               memory.
//   warp 2      scheduler: the key list of tile i, sorted by tile kind, with
//               the row mask and piece counts of each packed tile, into one
//               of two list buffers.
//   warps 4-7   softmax group A (key tiles 0, 2, 4, ... of a query tile),
//   warps 8-11  group B (1, 3, 5, ...): one row per thread, running max and
//               sum, P (bf16, or e4m3 four keys to a column) over its S;
//               then the epilogue of the tile: the two groups' partial
//               results merged (a split-key combine), normalised and stored.
// Tensor memory: S_A | S_B | O_A | O_B (512 columns).  The natural and slot
// forms pack the same tiles in the same order, so they give identical bits.
// Every wait is bounded; a wait that runs out records a timeout in the
// plan's status word and the CTA leaves without trapping.
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
constexpr int kThreads = 384;
constexpr int kListMax = 768;           // key-list entries a tile can pack
constexpr int kMaxBins = 128;           // packed tiles of edge pieces a list can hold
constexpr uint16_t kBad = 0xffffu;      // packed-list marker of an out-of-range entry
constexpr uint32_t kAll = 0xffffffffu;

template <int D, bool F8>
struct DraftCfg {
  static constexpr int kElem = F8 ? 1 : 2;         // bytes per element
  static constexpr int kChunkElems = 128 / kElem;  // elements per 128-byte swizzle row
  static constexpr int kChunks = D / kChunkElems;  // 128-byte swizzle panels
  static constexpr int kPanel = kTile * 128;
  static constexpr int kTileBytes = kTile * D * kElem;
  static constexpr int kKeysPerMma = 32 / kElem;   // K of one MMA: 16 (bf16) or 32 (e4m3)
  static constexpr int kPHalfCols = 16 * kElem;    // TMEM columns of 64 keys of P
  // K and V have rings of their own: K is needed a softmax earlier than V,
  // so it runs deeper; 8-bit tiles are half the size and both run deeper
  static constexpr int NK = F8 ? 4 : 3, NV = F8 ? 4 : 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTileBytes;
  static constexpr int kOffV = kOffK + NK * kTileBytes;
  static constexpr int kOffBar = kOffV + NV * kTileBytes;
  // q_full, q_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  // s_full[2], p_half[2], p_ready[2], o_final, o_free, list_full[2], list_empty[2],
  // stats_full[2]
  static constexpr int kNumBars = 2 + 2 * NK + 2 * NV + 2 + 2 + 2 + 2 + 2 + 2 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;     // tmem, abort
  static constexpr int kOffStats = kOffMisc + 16;             // [2][4][128] floats
  static constexpr int kOffLists = kOffStats + 2 * 4 * kTile * 4;
  // a list buffer: bin row masks (uint4), bin piece counts (uint32), the
  // entries (uint16), the header
  static constexpr int kOffBinVm = 0;
  static constexpr int kOffBinCnt = kMaxBins * 16;
  static constexpr int kOffEnt = kOffBinCnt + kMaxBins * 4;
  static constexpr int kOffHead = kOffEnt + kListMax * 2;
  static constexpr int kListBytes = kOffHead + 32;
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
  int slot;       // 1: [B, Hh, Npad, D] slot tensors, tile kt = slots 128 kt ..
  int64_t Npad;   //    (slot mode) slots per (b, head)
  int B, Hh, T, H, W, N, TW, TH, ph, pw;
  int64_t nblocks, ntiles, total_tiles;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int per_head;
  int64_t nlists;
  float scale, scale_log2;
  __nv_bfloat16* o;
  float* lse;
  const float* fp8_scales;  // 8-bit tiles: [3][B][Hh] scales of Q, K, V
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

__device__ __forceinline__ void end_sync() { asm volatile("bar.sync 2, 384;" ::: "memory"); }

// SLOT: slot tensors (p.slot); a template flag, so the natural-layout
// kernel carries none of the slot paths' code.
template <int D, bool F8, bool SLOT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_draft_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DraftParams p,
                      const __grid_constant__ DraftEdgeMaps em) {
  using Cfg = DraftCfg<D, F8>;
  static_assert(!F8 || D == 128, "8-bit tiles: D = 128");
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
  uint64_t* p_half = s_full + 2;          // [2]: keys 0..63 of P stored
  uint64_t* p_ready = p_half + 2;         // [2]: all of P stored
  uint64_t* o_final = p_ready + 2;
  uint64_t* o_free = o_final + 1;
  uint64_t* list_full = o_free + 1;       // [2]
  uint64_t* list_empty = list_full + 2;   // [2]
  uint64_t* stats_full = list_empty + 2;  // [2]: both groups' (max, sum) of a query tile
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);  // tmem, abort, skip
  float* stats = reinterpret_cast<float*>(smem + Cfg::kOffStats);
  auto list_base = [&](int buf) { return smem + Cfg::kOffLists + buf * Cfg::kListBytes; };
  auto list_entries = [&](int buf) {
    return reinterpret_cast<uint16_t*>(list_base(buf) + Cfg::kOffEnt);
  };
  auto list_head = [&](int buf) {
    return reinterpret_cast<ListHead*>(list_base(buf) + Cfg::kOffHead);
  };
  // bin b of a packed list: its row mask and its pieces per kind (one byte each)
  auto bin_vm = [&](int buf) { return reinterpret_cast<uint4*>(list_base(buf) + Cfg::kOffBinVm); };
  auto bin_cnt = [&](int buf) {
    return reinterpret_cast<uint32_t*>(list_base(buf) + Cfg::kOffBinCnt);
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
    mbar_init(&p_half[0], 128);
    mbar_init(&p_half[1], 128);
    mbar_init(&p_ready[0], 128);
    mbar_init(&p_ready[1], 128);
    mbar_init(o_final, 1);
    mbar_init(o_free, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&list_full[i], 32);
      mbar_init(&list_empty[i], 2 + 1 + 256);  // producers, MMA warp, softmax threads
      mbar_init(&stats_full[i], 256);
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
        bool packed = p.pk_on && n > 0 && n <= kListMax;
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
          // the bins of edge pieces, each with its row mask, computed once here
          // for the producers and the softmax groups
          int rr[3] = {ce[0], ce[1], ce[2]}, a[3];
          int nb = 0;
          uint4* bvm = bin_vm(buf);
          uint32_t* bcnt = bin_cnt(buf);
          while (rr[0] + rr[1] + rr[2] > 0 && nb < kMaxBins) {
            next_bin(p, rr, a);
            if (lane == 0) {
              uint32_t vm[4] = {0u, 0u, 0u, 0u};
              int off = 0;
              for (int e = 0; e < 3; ++e)
                for (int m = 0; m < a[e]; ++m) {
                  set_rows(vm, off, off + p.pk_rows[e]);
                  off += p.pk_step[e];
                }
              bvm[nb] = make_uint4(vm[0], vm[1], vm[2], vm[3]);
              bcnt[nb] = (uint32_t)a[0] | ((uint32_t)a[1] << 8) | ((uint32_t)a[2] << 16);
            }
            ++nb;
          }
          if (rr[0] + rr[1] + rr[2] > 0) {
            // more bins than the buffer holds: run this list unpacked (the
            // entries are read from col_idx again, in list order)
            packed = false;
          } else {
            npk = cF + nb;
          }
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
            mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
            if constexpr (SLOT) {
              const int row0 = (int)(((int64_t)b * p.Hh + h) * p.Npad + (int64_t)qt * kTile);
              for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_2d(sQ + c * Cfg::kPanel, &tmq, q_full, c * Cfg::kChunkElems, row0);
            } else {
              int x0, y0, fr;
              nat_coords(qt, b, x0, y0, fr);
              for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_5d(sQ + c * Cfg::kPanel, &tmq, q_full, c * Cfg::kChunkElems, h, x0, y0, fr);
            }
          }
          __syncwarp();
          issued_q = i + 1;
        }
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
            const uint32_t cnt = bin_cnt(buf)[j - hd.nF];
            const int a[3] = {(int)(cnt & 255u), (int)((cnt >> 8) & 255u), (int)(cnt >> 16)};
            if (elect_one()) {
              uint32_t bytes = 0;
#pragma unroll
              for (int e = 0; e < 3; ++e) bytes += a[e] * p.pk_rows[e] * 128 * Cfg::kChunks;
              mbar_arrive_expect_tx(&full[st], bytes);
              int off = 0;
#pragma unroll
              for (int e = 0; e < 3; ++e) {
                for (int m = 0; m < a[e]; ++m) {
                  const int kt = ent[pstart[e] + pptr[e] + m];
                  const CUtensorMap* mx = isK ? &em.k[p.pk_kind[e] - 1] : &em.v[p.pk_kind[e] - 1];
                  if constexpr (SLOT) {
                    // the piece's valid slots: a box of its exact size in the
                    // [tile][row][column] view of the slot tensor
                    const int tile = (int)(((int64_t)b * p.Hh + h) * p.nblocks + kt);
                    for (int c = 0; c < Cfg::kChunks; ++c)
                      tma_load_4d(dst + c * Cfg::kPanel + off * 128, mx, &full[st],
                                  c * Cfg::kChunkElems, 0, 0, tile);
                  } else {
                    int x0, y0, fr;
                    nat_coords(kt, b, x0, y0, fr);
                    for (int c = 0; c < Cfg::kChunks; ++c)
                      tma_load_5d(dst + c * Cfg::kPanel + off * 128, mx, &full[st],
                                  c * Cfg::kChunkElems, h, x0, y0, fr);
                  }
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
              mbar_arrive_expect_tx(&full[st], Cfg::kTileBytes);
              if constexpr (SLOT) {
                const int row0 = (int)(((int64_t)b * p.Hh + h) * p.Npad + (int64_t)kt * kTile);
                for (int c = 0; c < Cfg::kChunks; ++c)
                  tma_load_2d(dst + c * Cfg::kPanel, tmx, &full[st], c * Cfg::kChunkElems, row0);
              } else {
                int x0, y0, fr;
                nat_coords(kt, b, x0, y0, fr);
                for (int c = 0; c < Cfg::kChunks; ++c)
                  tma_load_5d(dst + c * Cfg::kPanel, tmx, &full[st], c * Cfg::kChunkElems, h, x0, y0, fr);
              }
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
      constexpr uint32_t idesc_qk = F8 ? idesc_e4m3(128, 128, 0) : idesc_bf16(128, 128, 0);
      constexpr uint32_t idesc_pv = F8 ? idesc_e4m3(128, D, 1) : idesc_bf16(128, D, 1);
      const uint64_t qd = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t vd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffV), Cfg::kPanel, 1024);
      auto issue_qk = [&](int st, uint32_t tdst) {
        const uint64_t kd = sdesc_add(kd0, st * Cfg::kTileBytes);  // K ring stage
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / Cfg::kKeysPerMma; ++kk) {
            // K step kk: 32 bytes along the 128-byte swizzle row, then the next panel
            const uint32_t off = (kk >> 2) * Cfg::kPanel + (kk & 3) * 32;
            if constexpr (F8)
              mma_ss_f8(tdst, sdesc_add(qd, off), sdesc_add(kd, off), idesc_qk, kk > 0);
            else
              mma_ss(tdst, sdesc_add(qd, off), sdesc_add(kd, off), idesc_qk, kk > 0);
          }
        }
        __syncwarp();
      };
      // O_g (+)= P(keys 64 * half .. + 63) . V(same keys)
      auto issue_pv = [&](int st, int g, int half, uint32_t acc) {
        const uint64_t vd = sdesc_add(vd0, st * Cfg::kTileBytes + half * 64 * 128);
        const uint32_t tP = tbase + g * 128 + 64 + half * Cfg::kPHalfCols;
        const uint32_t tO = tbase + 256 + g * 128;
        if (elect_one()) {
          // K step kk: the next kKeysPerMma keys = 8 TMEM columns of P and
          // kKeysPerMma 128-byte rows of V
#pragma unroll
          for (int kk = 0; kk < 64 / Cfg::kKeysPerMma; ++kk) {
            const uint64_t bd = sdesc_add(vd, kk * Cfg::kKeysPerMma * 128);
            const uint32_t on = (acc | (uint32_t)half | (uint32_t)kk) != 0;
            if constexpr (F8)
              mma_ts_f8(tO, tP + kk * 8, bd, idesc_pv, on);
            else
              mma_ts(tO, tP + kk * 8, bd, idesc_pv, on);
          }
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
      // QK of tile t (ring position jj + t) into the S buffer of its group
      auto qk = [&](int t) {
        const int64_t q = jj + t;
        const int st = (int)(q % Cfg::NK);
        if (!wait(&k_full[st], (uint32_t)((q / Cfg::NK) & 1))) return false;
        tc_fence_after();
        issue_qk(st, tbase + (t & 1) * 128);
        commit(&s_full[t & 1]);
        commit(&k_empty[st]);
        return true;
      };
      for (int64_t i = 0; alive && i < my_tiles; ++i) {
        const int buf = (int)(i & 1);
        if (!wait(&list_full[buf], (uint32_t)((i >> 1) & 1))) break;
        const int n = list_head(buf)->n;
        __syncwarp();
        if (lane == 0) mbar_arrive(&list_empty[buf]);
        if (!wait(q_full, (uint32_t)(i & 1))) break;
        tc_fence_after();
        // group g takes tiles g, g + 2, ...; each group's next QK follows its
        // own PV, so S of tile j+2 is ready as soon as PV of tile j is done
        if (n > 0 && !qk(0)) break;
        if (n > 1 && !qk(1)) break;
        if (n <= 2) commit(q_empty);  // Q no longer read once those QKs complete
        for (int j = 0; j < n; ++j) {
          const int g = j & 1;
          const int64_t q0 = jj + j;
          const int st = (int)(q0 % Cfg::NV);
          const uint32_t ph = (uint32_t)(pcount[g] & 1);
          if (!wait(&p_half[g], ph) || !wait(&v_full[st], (uint32_t)((q0 / Cfg::NV) & 1))) {
            alive = false;
            break;
          }
          // the previous tile's output must be out of tensor memory before
          // this tile's first PV overwrites O
          if (j == 0 && i > 0 && !wait(o_free, (uint32_t)((i - 1) & 1))) { alive = false; break; }
          tc_fence_after();
          issue_pv(st, g, 0, j >= 2);
          if (!wait(&p_ready[g], ph)) { alive = false; break; }
          ++pcount[g];
          tc_fence_after();
          issue_pv(st, g, 1, 1);
          commit(&v_empty[st]);
          if (j + 2 < n) {
            if (!qk(j + 2)) { alive = false; break; }
            if (j + 3 == n) commit(q_empty);
          }
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
    float sl2 = p.scale_log2;
    float thr = 8.0f / sl2;  // rescale O when the max grows by more than 2^8
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
      // 8-bit tiles: S holds q8.k8, the scores are S * sq * sk; O holds
      // P.v8, the values are O * sv
      float sqk = 1.f, sv = 1.f;
      if (F8) {
        sqk = p.fp8_scales[(int64_t)b * p.Hh + h] * p.fp8_scales[((int64_t)p.B + b) * p.Hh + h];
        sv = p.fp8_scales[(2 * (int64_t)p.B + b) * p.Hh + h];
        sl2 = p.scale_log2 * sqk;
        thr = 8.0f / sl2;
      }
      RowState rs;
      for (int j = g; j < n; j += 2) {
        uint32_t vm[4] = {0u, 0u, 0u, 0u};
        if (hd.packed && j >= hd.nF) {
          const uint4 b = bin_vm(buf)[j - hd.nF];
          vm[0] = b.x;
          vm[1] = b.y;
          vm[2] = b.z;
          vm[3] = b.w;
        } else if (hd.packed) {
          // a full tile (every slot holds a token) unless the entry was out of range
          const uint32_t f = ent[j] != kBad ? kAll : 0u;
          vm[0] = vm[1] = vm[2] = vm[3] = f;
        } else {
          int kt;
          bool ok;
          {
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
        float corr;
        uint64_t neg_ms2;
        // most key tiles are full: they take a copy of the step without masking
        const bool need = (vm[0] & vm[1] & vm[2] & vm[3]) == kAll
                              ? softmax_max<128, false>(s, vm, rs, sl2, thr, corr, neg_ms2)
                              : softmax_max<128, true>(s, vm, rs, sl2, thr, corr, neg_ms2);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        if constexpr (F8) {
          uint32_t pk[16];
          softmax_exp_e4m3<0, 128>(s, sl2, neg_ms2, pk, acc);
          tmem_st16(tS + 64, pk);
        } else {
          uint32_t pk[32];
          softmax_exp<0, 64>(s, sl2, neg_ms2, pk, acc);
          tmem_st32(tS + 64, pk);
        }
        // O of this group holds every earlier PV of the group in this query
        // tile (S(j) was written after the group's previous PV); it is
        // rescaled before this tile's first PV, once half of s is no longer
        // live
        if (j >= 2 && __any_sync(kAll, need)) tmem_scale<D>(tO, corr);
        tc_fence_before();
        mbar_arrive(&p_half[g]);
        if constexpr (F8) {
          uint32_t pk[16];
          softmax_exp_e4m3<64, 128>(s, sl2, neg_ms2, pk, acc);
          tmem_st16(tS + 64 + Cfg::kPHalfCols, pk);
        } else {
          uint32_t pk[32];
          softmax_exp<64, 64>(s, sl2, neg_ms2, pk, acc);
          tmem_st32(tS + 64 + Cfg::kPHalfCols, pk);
        }
        softmax_sum(rs, acc);
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
      // statistics buffers alternate between query tiles: each group reads
      // tile i's before it reaches tile i+1's barrier, so tile i+2 may
      // overwrite them
      float* st = stats + (i & 1) * 4 * kTile;
      st[(2 * g) * kTile + row] = rs.m;
      st[(2 * g + 1) * kTile + row] = rs.l;
      // a bounded wait, not a named barrier: a group that gave up on an
      // earlier wait must not leave the other one waiting for good
      mbar_arrive(&stats_full[i & 1]);
      if (!__all_sync(kAll, bounded_wait(&stats_full[i & 1], (uint32_t)((i >> 1) & 1), wc))) {
        alive = false;
        break;
      }
      const float mA = st[row], lA = st[kTile + row];
      const float mB = st[2 * kTile + row], lB = st[3 * kTile + row];
      const int nA = (n + 1) / 2, nB = n / 2;
      const float m = fmaxf(mA, mB);
      const float a = (nA > 0 && mA != -INFINITY) ? ex2_approx((mA - m) * sl2) : 0.f;
      const float bb = (nB > 0 && mB != -INFINITY) ? ex2_approx((mB - m) * sl2) : 0.f;
      const float l = lA * a + lB * bb;
      bool qvalid;
      int64_t orow, lrow;
      if constexpr (SLOT) {
        // slot tensors: row `row` of tile qt; an empty slot is written as 0
        // (LSE -inf) like every slot of the layout
        const uint4 tq = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + qt);
        const uint32_t qw = (row < 32) ? tq.x : (row < 64) ? tq.y : (row < 96) ? tq.z : tq.w;
        qvalid = (qw >> (row & 31)) & 1u;
        orow = ((int64_t)b * p.Hh + h) * p.Npad + (int64_t)qt * kTile + row;
        lrow = orow;
      } else {
        // slot (y, x) of tile (t, i, j) is token (t, y0 + y, x0 + x); slots
        // past the grid's right or bottom edge hold no token
        int x0, y0, fr;
        nat_coords(qt, b, x0, y0, fr);
        const int ay = (int)p.div_pw.div((uint32_t)row);
        const int yy = y0 + ay, xx = x0 + (row - ay * p.pw);
        qvalid = ay < p.ph && yy < p.H && xx < p.W;
        const int t = fr - b * p.T;
        const int64_t ntok = ((int64_t)t * p.H + yy) * p.W + xx;
        orow = ((int64_t)b * p.N + ntok) * p.Hh + h;
        lrow = ((int64_t)b * p.Hh + h) * p.N + ntok;
      }
      const bool write = qvalid || SLOT;
      const bool has = n > 0 && qvalid && l > 0.f;
      const float inv_l = has ? sv / l : 0.f;
      const float wa = a * inv_l, wb = bb * inv_l;
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
          w16[e] = pack_bf16x2(v0, v1);
        }
        if (write) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[c * 4 + e] = make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2], w16[4 * e + 3]);
        }
      }
      if (g == 0 && p.lse && write) p.lse[lrow] = has ? m * (p.scale * sqk) + logf(l) : -INFINITY;
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

// Natural layout [B, N, Hh, D] as 5-D {D, Hh, W, H, B*T}; boxes of one
// 128-byte row of channels (64 bf16 or 128 e4m3) x 1 head x box_w x box_h x
// 1 frame, 128-byte swizzle; boxes reaching past W or H read zeros.
bool make_draft_tmap(CUtensorMap* m, const void* ptr, const Geometry& g, int box_w, int box_h,
                     bool e4m3 = false) {
  auto fn = draft_encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = e4m3 ? 1 : 2;
  const cuuint64_t row = (cuuint64_t)g.Hh * g.D * esz;
  cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.Hh, (cuuint64_t)g.W, (cuuint64_t)g.H,
                        (cuuint64_t)g.B * g.T};
  cuuint64_t strides[4] = {(cuuint64_t)g.D * esz, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {(cuuint32_t)(128 / esz), 1, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Slot tensors [B, Hh, Npad, D] bf16 as a 2-D [B*Hh*Npad, D] tensor; boxes of
// 64 channels x 128 slots, 128-byte swizzle.
bool make_slot_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int D) {
  auto fn = draft_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Slot tensors of a TILE plan (128 slots = one ph x pw tile, row-major) as a
// 4-D [B*Hh*nblocks][ph][pw][D] tensor; boxes of 64 channels x box_w x box_h,
// 128-byte swizzle: the valid slots of an edge tile, in row-major order.
bool make_slot_edge_tmap(CUtensorMap* m, const void* ptr, const Geometry& g, int box_w, int box_h) {
  auto fn = draft_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.pw, (cuuint64_t)g.ph,
                        (cuuint64_t)g.B * g.Hh * g.nblocks};
  cuuint64_t strides[3] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.pw * g.D * 2,
                           (cuuint64_t)kTile * g.D * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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

template <int D, bool F8 = false>
cudaError_t launch_draft_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const DraftParams& p, const DraftEdgeMaps& em, cudaStream_t st) {
  using Cfg = DraftCfg<D, F8>;
  auto kern = p.slot ? attn_draft_kernel<D, F8, true> : attn_draft_kernel<D, F8, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(p.total_tiles, draft_sm_count());
  kern<<<(unsigned)grid, kThreads, Cfg::kSmem, st>>>(q, k, v, p, em);
  return cudaGetLastError();
}

}  // namespace



bsa_status launch_attn_draft(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                             const int32_t* row_ptr, const int32_t* col_idx, int per_head,
                             float scale, void* o, float* lse, cudaStream_t st, bool slot,
                             const float* fp8_scales) {
  const bool f8 = fp8_scales != nullptr;
  const Geometry& g = plan.g;
  CUtensorMap tq, tk, tv;
  if (slot) {
    if (g.block != kTile)
      return set_error(BSA_ERR_UNSUPPORTED, "slot-layout persistent attention needs 128-slot blocks");
    const int64_t rows = (int64_t)g.B * g.Hh * g.Npad;
    if (rows >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "B*Hh*Npad must be < 2^31");
    if (!make_slot_tmap(&tq, q, rows, g.D) || !make_slot_tmap(&tk, k, rows, g.D) ||
        !make_slot_tmap(&tv, v, rows, g.D))
      return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (2-D) failed");
  } else {
    if (g.layout != BSA_LAYOUT_TILE || g.block != kTile)
      return set_error(BSA_ERR_UNSUPPORTED,
                       "natural-layout attention needs a TILE plan with pool_h * pool_w = 128");
    if (f8 && g.D != 128) return set_error(BSA_ERR_UNSUPPORTED, "e4m3 attention supports D = 128");
    if ((int64_t)g.B * g.T * g.P * g.Hh >= (1ll << 31))
      return set_error(BSA_ERR_UNSUPPORTED, "B*N*Hh must be < 2^31");
    if ((int64_t)g.B * g.T >= (1ll << 31))
      return set_error(BSA_ERR_UNSUPPORTED, "B*T must be < 2^31");
    if (!make_draft_tmap(&tq, q, g, g.pw, g.ph, f8) || !make_draft_tmap(&tk, k, g, g.pw, g.ph, f8) ||
        !make_draft_tmap(&tv, v, g, g.pw, g.ph, f8))
      return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (5-D) failed");
  }
  DraftParams p{};  // every field zero (the divisors 1) until set below
  p.slot = slot ? 1 : 0;
  p.Npad = g.Npad;
  p.fp8_scales = fp8_scales;
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
  DraftEdgeMaps em;
  memset(&em, 0, sizeof(em));
  if (slot && g.layout != BSA_LAYOUT_TILE) {
    // key tiles as stored (empty slots masked), no packing; the tile-grid
    // divisors are unused
    p.div_tile_frame = FastDiv(1u);
    p.div_TW = FastDiv(1u);
    p.div_pw = FastDiv(1u);
    const cudaError_t e = g.D == 128 ? launch_draft_t<128>(tq, tk, tv, p, em, st)
                                     : launch_draft_t<64>(tq, tk, tv, p, em, st);
    if (e != cudaSuccess) return cuda_error(e, "draft attention launch");
    return BSA_OK;
  }
  // the tile layout (natural tensors or their slots): edge tiles packed
  p.div_tile_frame = FastDiv((uint32_t)(g.TH * g.TW));
  p.div_TW = FastDiv((uint32_t)g.TW);
  p.div_pw = FastDiv((uint32_t)g.pw);
  int kind[3] = {0, 0, 0}, rows[3] = {0, 0, 0}, bw[3] = {0, 0, 0}, bh[3] = {0, 0, 0};
  const int nk = edge_kinds(g, kind, rows, bw, bh);
  if (nk > 0 && g.nblocks < 32768) {
    for (int i = 0; i < nk; ++i) {
      p.pk_kind[i] = kind[i];
      p.pk_rows[i] = rows[i];
      p.pk_step[i] = (rows[i] + 7) / 8 * 8;
      const bool ok = slot ? make_slot_edge_tmap(&em.k[kind[i] - 1], k, g, bw[i], bh[i]) &&
                                 make_slot_edge_tmap(&em.v[kind[i] - 1], v, g, bw[i], bh[i])
                           : make_draft_tmap(&em.k[kind[i] - 1], k, g, bw[i], bh[i], f8) &&
                                 make_draft_tmap(&em.v[kind[i] - 1], v, g, bw[i], bh[i], f8);
      if (!ok) return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled (edge boxes) failed");
    }
    p.pk_on = 1;
  }
  const cudaError_t e = f8 ? launch_draft_t<128, true>(tq, tk, tv, p, em, st)
                       : g.D == 128 ? launch_draft_t<128>(tq, tk, tv, p, em, st)
                                    : launch_draft_t<64>(tq, tk, tv, p, em, st);
  if (e != cudaSuccess) return cuda_error(e, "draft attention launch");
  return BSA_OK;
}

}  // namespace bsa
