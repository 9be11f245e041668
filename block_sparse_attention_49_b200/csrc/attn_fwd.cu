// Block-sparse softmax attention forward on sm_100a tensor cores.
//
// What it computes ("LVSA: Training-Free Sparse Attention for Long Video
// Diffusion", section 2: attention restricted to the blocks of the frame set
// A(t); Draft Attention article: the sparse mask guides full-resolution
// block-sparse attention): for every query slot, softmax(scale * q.k) over
// the non-empty key slots of the key blocks its query block may attend,
// weighted sum of their values; plus the log-sum-exp.
//
// How (one CTA per 128-slot query tile; 12 warps):
//   warp 0      TMA producer: the Q tile once, then K and V of every listed
//               key tile into an NS-deep shared-memory ring (128-byte swizzle).
//   warp 1      MMA issuer (the whole warp runs the loop, an elected lane
//               issues): S = Q K^T into tensor memory, then O += P V with P
//               read from tensor memory.
//   warps 4-7   softmax group A: key tiles 0, 2, 4, ... of the list;
//   warps 8-11  softmax group B: key tiles 1, 3, 5, ...
// Each group owns one S buffer and one O accumulator in tensor memory
// (S_A | S_B | O_A | O_B = 512 columns) and keeps its own running max and
// sum, so the two groups never wait for each other inside the loop: while one
// group's softmax runs, the tensor cores work on the other group's tiles.
// Each thread owns one query row (one TMEM lane): it reads its S row, masks
// empty or disallowed keys, writes P as bf16 over the upper half of its S
// buffer, and rescales its O only when its running max grew by more than 2^8
// (numerator and denominator share the stale max, so the result is exact).
// At the end the two partial results are merged with their maxima and sums,
// as in a split-key combine, normalised and stored.
// Every wait is bounded; a wait that runs out records a timeout in the
// plan's status word and the CTA leaves without trapping.
//
// FINE (template flag): blocks smaller than 128 slots; each row walks its own
// CSR row.  Lists of 128-slot blocks run elsewhere: per-head lists and the
// natural-layout and 8-bit draft paths on the persistent kernel
// (attn_draft.cu), lists shared by every head on the paired kernel
// (attn_pair.cu); this kernel keeps shared lists too long for the latter.
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

constexpr int kTile = 128;          // query / key tile (slots)
constexpr int kThreads = 384;
constexpr int kFineMaxTiles = 2048; // key tiles addressable by the sub-tile-block path
constexpr uint32_t kFull = 0xffffffffu;

template <int D, bool FINE>
struct AttnCfg {
  static constexpr int kChunks = D / 64;             // 128-byte-wide swizzle panels
  static constexpr int kPanel = kTile * 128;
  static constexpr int kQBytes = kTile * D * 2;
  static constexpr int kKVBytes = kTile * D * 2;
  static constexpr int kKeysPerMma = 16;             // K of one bf16 MMA
  static constexpr int NS = (D == 128) ? (FINE ? 2 : 3) : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + NS * kKVBytes;
  static constexpr int kOffBar = kOffV + NS * kKVBytes;
  static constexpr int kNumBars = 1 + 3 * NS + 2 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffList = kOffMisc + 16;
  // FINE: the union of key tiles (uint16)
  static constexpr int kOffBitmap = kOffList + (FINE ? kFineMaxTiles * 2 : 0);
  static constexpr int kBytes = kOffBitmap + (FINE ? kFineMaxTiles / 8 : 0);
  static constexpr int kSmem = kBytes + 1024;  // room to align the base to 1024
  static constexpr uint32_t kTmemCols = 512;   // S_A | S_B | O_A | O_B
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(4 * kTile * 4 <= kKVBytes, "epilogue statistics fit in a K stage");
};

struct AttnParams {
  int Hh;
  int block;          // slots per block of the block list
  int64_t Npad;       // slots per (b, head)
  int64_t nblocks;    // blocks per (b, head)
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int per_head;
  int64_t nlists;     // block lists in the CSR: B*Hh if per_head else 1
  float scale;        // softmax scale applied to q.k
  float scale_log2;   // scale * log2(e)
  __nv_bfloat16* o;
  float* lse;
  const uint32_t* tile_valid;  // [ntiles][4]
  unsigned int* status;
  uint64_t wait_limit_ns;
};

// Set bits [lo, lo+len) of a 128-bit mask; lo is a multiple of len, len | 128.
__device__ __forceinline__ void set_bits(uint32_t (&m)[4], int lo, int len) {
  if (len >= 32) {
    for (int x = lo; x < lo + len; x += 32) m[x >> 5] = kFull;
  } else {
    m[lo >> 5] |= ((1u << len) - 1u) << (lo & 31);
  }
}

__device__ __forceinline__ void softmax_groups_sync() {
  asm volatile("bar.sync 1, 256;" ::: "memory");  // warps 4-11
}

// Final CTA barrier, reached by every warp from its own role branch.
__device__ __forceinline__ void cta_end_sync() {
  asm volatile("bar.sync 2, 384;" ::: "memory");
}

template <int D, bool FINE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const AttnParams p) {
  using Cfg = AttnCfg<D, FINE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + Cfg::NS;
  uint64_t* kv_empty = v_full + Cfg::NS;
  uint64_t* s_full = kv_empty + Cfg::NS;  // [2]: S_A, S_B written
  uint64_t* p_half = s_full + 2;          // [2]: keys 0..63 of P_A, P_B written
  uint64_t* p_ready = p_half + 2;         // [2]: P_A, P_B written (128 arrivals each)
  uint64_t* o_final = p_ready + 2;        // every MMA done
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);  // tmem, abort, count, skip
  uint16_t* tlist = reinterpret_cast<uint16_t*>(smem + Cfg::kOffList);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + Cfg::kOffBitmap);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh_row = ((int64_t)b * p.Hh + h) * p.Npad;
  const int64_t list = p.per_head ? (int64_t)b * p.Hh + h : 0;
  const WaitCtx wc{p.status, reinterpret_cast<volatile int*>(&misc[1]), p.wait_limit_ns};

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < Cfg::NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
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
    // a timeout recorded by an earlier CTA (or call) stops the rest of the grid
    misc[3] = (*reinterpret_cast<volatile unsigned int*>(p.status) & kStatusTimeout) ? 1u : 0u;
    fence_mbar_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  __syncthreads();
  if (misc[3]) return;
  if (warp == 1) {
    tmem_alloc(&misc[0], Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (FINE) {
    for (int i = threadIdx.x; i < kFineMaxTiles / 32; i += kThreads) bitmap[i] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  // ------------------------------------------------ key tiles of this query tile
  int64_t rs = 0;
  int n = 0;
  const int64_t nnz = p.row_ptr[p.nlists * p.nblocks];  // entries of col_idx
  if (!FINE) {
    const int64_t r = list * p.nblocks + qt;  // block == tile
    rs = p.row_ptr[r];
    const int64_t re = p.row_ptr[r + 1];
    if (re < rs || rs < 0 || re > nnz) {
      if (threadIdx.x == 0) atomicOr(p.status, kStatusBadBlocklist);
    } else {
      n = (int)(re - rs);
    }
  } else {
    // union over the query blocks of this tile of the key tiles they touch
    const int per = kTile / p.block;
    const int64_t qb0 = (int64_t)qt * per;
    const int64_t qb1 = min(qb0 + per, p.nblocks);
    for (int64_t qb = qb0 + warp; qb < qb1; qb += kThreads / 32) {
      const int64_t r = list * p.nblocks + qb;
      const int64_t a = max(p.row_ptr[r], 0), e = min((int64_t)p.row_ptr[r + 1], nnz);
      for (int64_t i = a + lane; i < e; i += 32) {
        const int c = p.col_idx[i];
        if (c >= 0 && c < p.nblocks) {
          const int tile = (int)(((int64_t)c * p.block) >> 7);
          atomicOr(&bitmap[tile >> 5], 1u << (tile & 31));
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cnt = 0;
      for (int w = 0; w < kFineMaxTiles / 32; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
          const int bpos = __ffs(bits) - 1;
          bits &= bits - 1;
          tlist[cnt++] = (uint16_t)(w * 32 + bpos);
        }
      }
      misc[2] = cnt;
    }
    __syncthreads();
    n = (int)misc[2];
  }

  auto tile_of = [&](int j, bool& ok) -> int {
    if (FINE) {
      ok = true;
      return tlist[j];
    }
    const int c = __ldg(p.col_idx + rs + j);
    ok = (c >= 0 && (int64_t)c < p.nblocks);
    return ok ? c : 0;
  };

  if (warp < 4) {
    // producer, MMA issuer and two idle warps: few registers
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
    if (warp == 0 && n > 0) {
      // -------------------------------------------------------- TMA producer
      // the whole warp runs the loop (warp-uniform operands); one lane issues
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_2d(sQ + c * Cfg::kPanel, &tmq, q_full, c * 64,
                      (int)(bh_row + (int64_t)qt * kTile));
      }
      __syncwarp();
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % Cfg::NS;
        const uint32_t ph = (j / Cfg::NS) & 1;
        if (!__all_sync(kFull, bounded_wait(&kv_empty[st], ph ^ 1, wc))) break;
        bool ok;
        const int kt = tile_of(j, ok);
        const int krow = (int)(bh_row + (int64_t)kt * kTile);
        if (elect_one()) {
          if (!ok) atomicOr(p.status, kStatusBadBlocklist);
          uint8_t* sK = smem + Cfg::kOffK + st * Cfg::kKVBytes;
          uint8_t* sV = smem + Cfg::kOffV + st * Cfg::kKVBytes;
          mbar_arrive_expect_tx(&k_full[st], Cfg::kKVBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_2d(sK + c * Cfg::kPanel, &tmk, &k_full[st], c * 64, krow);
          mbar_arrive_expect_tx(&v_full[st], Cfg::kKVBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_2d(sV + c * Cfg::kPanel, &tmv, &v_full[st], c * 64, krow);
        }
        __syncwarp();
        issued = j + 1;
      }
      if (*wc.abort) {
        // leave no copy in flight: wait (bounded, ignoring the abort flag)
        // for the loads still owned by the ring
        volatile int no_abort = 0;
        const WaitCtx drain{p.status, &no_abort, p.wait_limit_ns};
        bounded_wait(q_full, 0, drain);
        for (int j = max(0, issued - Cfg::NS); j < issued; ++j) {
          bounded_wait(&k_full[j % Cfg::NS], (j / Cfg::NS) & 1, drain);
          bounded_wait(&v_full[j % Cfg::NS], (j / Cfg::NS) & 1, drain);
        }
      }
      __syncwarp();
    } else if (warp == 1 && n > 0) {
      // -------------------------------------------------------- MMA issuer
      // the whole warp runs the loop (descriptors stay warp-uniform); the
      // elected lane issues the tcgen05 instructions
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, 1);
      const uint64_t qd = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t vd0 = sdesc_sw128(smem_u32(smem + Cfg::kOffV), Cfg::kPanel, 1024);
      auto issue_qk = [&](int st, uint32_t tdst) {
        const uint64_t kd = sdesc_add(kd0, st * Cfg::kKVBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / Cfg::kKeysPerMma; ++kk) {
            // K step kk: 32 bytes along the 128-byte swizzle row, then the next panel
            const uint32_t off = (kk >> 2) * Cfg::kPanel + (kk & 3) * 32;
            mma_ss(tdst, sdesc_add(qd, off), sdesc_add(kd, off), idesc_qk, kk > 0);
          }
        }
        __syncwarp();
      };
      // O_g (+)= P(keys 64 * half .. + 63) . V(same keys)
      auto issue_pv_half = [&](int st, int g, int half, uint32_t acc) {
        const uint64_t vd = sdesc_add(vd0, st * Cfg::kKVBytes + half * 64 * 128);
        const uint32_t tP = tbase + g * 128 + 64 + half * 32, tO = tbase + 256 + g * 128;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tO, tP + kk * 8, sdesc_add(vd, kk * 16 * 128), idesc_pv,
                   (acc | (uint32_t)half | (uint32_t)kk) != 0);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) mma_commit(bar);
        __syncwarp();
      };
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(kFull, bounded_wait(bar, parity, wc));
      };
      // group g takes tiles g, g + 2, ...; QK of tile j+2 follows PV of
      // tile j, so each group's next S is ready as soon as its PV is done;
      // P is handed over in two halves
      auto qk = [&](int t) {
        const int st = t % Cfg::NS;
        if (!wait(&k_full[st], (t / Cfg::NS) & 1)) return false;
        tc_fence_after();
        issue_qk(st, tbase + (t & 1) * 128);
        commit(&s_full[t & 1]);
        return true;
      };
      bool alive = wait(q_full, 0) && qk(0) && (n < 2 || qk(1));
      for (int j = 0; alive && j < n; ++j) {
        const int g = j & 1, st = j % Cfg::NS;
        if (!wait(&p_half[g], (j >> 1) & 1) || !wait(&v_full[st], (j / Cfg::NS) & 1)) break;
        tc_fence_after();
        issue_pv_half(st, g, 0, j >= 2);
        if (!wait(&p_ready[g], (j >> 1) & 1)) break;
        tc_fence_after();
        issue_pv_half(st, g, 1, 1);
        commit(&kv_empty[st]);
        if (j + 2 < n && !qk(j + 2)) break;
      }
      commit(o_final);
    }
    cta_end_sync();
    if (warp == 1) {
      // every tensor-memory read of the softmax groups is done: free TMEM
      tc_fence_after();
      tmem_dealloc(tbase, Cfg::kTmemCols);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    // ---------------------------------------------------------- softmax groups
    const int g = (warp >= 8) ? 1 : 0;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + g * 128 + lane_off;
    const uint32_t tO = tbase + 256 + g * 128 + lane_off;
    const float sl2 = p.scale_log2;
    const float thr = 8.0f / sl2;  // rescale O when the max grows by more than 2^8
    RowState rs;
    int64_t fptr = 0, fend = 0;
    int fprev = -1;
    if (FINE) {
      const int64_t qb = (int64_t)qt * (kTile / p.block) + row / p.block;
      if (qb < p.nblocks) {
        const int64_t r = list * p.nblocks + qb;
        fptr = p.row_ptr[r];
        fend = p.row_ptr[r + 1];
        if (fend < fptr || fptr < 0 || fend > nnz) {
          if (g == 0) atomicOr(p.status, kStatusBadBlocklist);
          fend = fptr;
        }
      }
    }
    bool alive = true;
    for (int j = g; j < n; j += 2) {
      uint32_t vm[4] = {0u, 0u, 0u, 0u};
      {
        bool ok;
        const int kt = tile_of(j, ok);
        const uint4 tv = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + kt);
        vm[0] = ok ? tv.x : 0u;
        vm[1] = ok ? tv.y : 0u;
        vm[2] = ok ? tv.z : 0u;
        vm[3] = ok ? tv.w : 0u;
      }
      if (FINE) {
        bool ok;
        const int kt = tile_of(j, ok);
        // this row's allowed blocks inside key tile kt (entries of tiles
        // handled by the other group are passed over)
        uint32_t am[4] = {0u, 0u, 0u, 0u};
        while (fptr < fend) {
          const int c = __ldg(p.col_idx + fptr);
          if (c < 0 || c >= p.nblocks || c <= fprev) {  // out of range or not ascending
            atomicOr(p.status, kStatusBadBlocklist);
            ++fptr;
            continue;
          }
          const int64_t s0 = (int64_t)c * p.block;
          const int ct = (int)(s0 >> 7);
          if (ct > kt) break;
          if (ct == kt) set_bits(am, (int)(s0 & 127), p.block);
          fprev = c;
          ++fptr;
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) vm[w] &= am[w];
      }
      if (!__all_sync(kFull, bounded_wait(&s_full[g], (j >> 1) & 1, wc))) {
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
      // full key tiles take a copy of the step without masking
      const bool need = (vm[0] & vm[1] & vm[2] & vm[3]) == kFull
                            ? softmax_max<128, false>(s, vm, rs, sl2, thr, corr, neg_ms2)
                            : softmax_max<128, true>(s, vm, rs, sl2, thr, corr, neg_ms2);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      {
        uint32_t pk[32];
        softmax_exp<0, 64>(s, sl2, neg_ms2, pk, acc);
        tmem_st32(tS + 64, pk);
      }
      // O of this group holds every earlier PV of the group (S(j) was
      // written after the group's previous PV); it is rescaled before this
      // tile's first PV, once half of s is no longer live
      if (j >= 2 && __any_sync(kFull, need)) tmem_scale<D>(tO, corr);
      tc_fence_before();
      mbar_arrive(&p_half[g]);
      {
        uint32_t pk[32];
        softmax_exp<64, 64>(s, sl2, neg_ms2, pk, acc);
        tmem_st32(tS + 96, pk);
      }
      softmax_sum(rs, acc);
      tc_fence_before();
      mbar_arrive(&p_ready[g]);
    }
    // ---------------------------------------------------------- epilogue
    if (alive && n > 0) {
      alive = __all_sync(kFull, bounded_wait(o_final, 0, wc));
      tc_fence_after();
    }
    // exchange (max, sum) of the two groups through a free K stage
    float* stats = reinterpret_cast<float*>(smem + Cfg::kOffK);  // [4][128]: mA lA mB lB
    stats[(2 * g) * kTile + row] = rs.m;
    stats[(2 * g + 1) * kTile + row] = rs.l;
    softmax_groups_sync();
    const float mA = stats[row], lA = stats[kTile + row];
    const float mB = stats[2 * kTile + row], lB = stats[3 * kTile + row];
    const int nA = (n + 1) / 2, nB = n / 2;  // tiles each group processed
    const float m = fmaxf(mA, mB);
    const float a = (nA > 0 && mA != -INFINITY) ? ex2_approx((mA - m) * sl2) : 0.f;
    const float bb = (nB > 0 && mB != -INFINITY) ? ex2_approx((mB - m) * sl2) : 0.f;
    const float l = lA * a + lB * bb;
    const uint4 tq = __ldg(reinterpret_cast<const uint4*>(p.tile_valid) + qt);
    const uint32_t qw = (row < 32) ? tq.x : (row < 64) ? tq.y : (row < 96) ? tq.z : tq.w;
    const bool qvalid = (qw >> (row & 31)) & 1u;
    const bool has = alive && n > 0 && qvalid && l > 0.f;
    const float inv_l = has ? 1.f / l : 0.f;
    const float wa = a * inv_l, wb = bb * inv_l;
    const int64_t orow = bh_row + (int64_t)qt * kTile + row;  // slot row = LSE index
    // group g stores columns [g*D/2, (g+1)*D/2) of its rows
    uint4* dst = reinterpret_cast<uint4*>(p.o + orow * D + g * (D / 2));
    const uint32_t oA = tbase + 256 + lane_off + g * (D / 2);
    const uint32_t oB = tbase + 384 + lane_off + g * (D / 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t xa[32], xb[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) xa[i] = xb[i] = 0u;
      if (alive && nA > 0) tmem_ld32(oA + c * 32, xa);
      if (alive && nB > 0) tmem_ld32(oB + c * 32, xb);
      uint32_t w16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v0 = has ? __uint_as_float(xa[2 * i]) * wa + __uint_as_float(xb[2 * i]) * wb : 0.f;
        const float v1 =
            has ? __uint_as_float(xa[2 * i + 1]) * wa + __uint_as_float(xb[2 * i + 1]) * wb : 0.f;
        w16[i] = pack_bf16x2(v0, v1);
      }
      {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[c * 4 + i] = make_uint4(w16[4 * i], w16[4 * i + 1], w16[4 * i + 2], w16[4 * i + 3]);
      }
    }
    if (g == 0 && p.lse) p.lse[orow] = has ? m * p.scale + logf(l) : -INFINITY;
    tc_fence_before();
    cta_end_sync();
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [rows, D] bf16 row-major, 64 x 128 boxes, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool FINE>
cudaError_t launch_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                     const AttnParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = AttnCfg<D, FINE>;
  auto kern = attn_fwd_kernel<D, FINE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, Cfg::kSmem, st>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

namespace {

AttnParams make_params(const bsa_plan_s& plan, const int32_t* row_ptr, const int32_t* col_idx,
                       int per_head, float scale, void* o, float* lse) {
  const Geometry& g = plan.g;
  AttnParams p;
  p.Hh = g.Hh;
  p.block = g.block;
  p.Npad = g.Npad;
  p.nblocks = g.nblocks;
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
  return p;
}

}  // namespace

// Edge kinds of a TILE plan's grid: right (kind 1, the last tile column when
// pool_w does not divide W), bottom (2) and corner (3), sorted by size
// (rows), largest first; their box width and height.
int edge_kinds(const Geometry& g, int kind[3], int rows[3], int bw[3], int bh[3]) {
  const int wR = g.W - (g.TW - 1) * g.pw, hB = g.H - (g.TH - 1) * g.ph;
  int n = 0;
  auto add = [&](int k, int w, int h) {
    kind[n] = k;
    rows[n] = w * h;
    bw[n] = w;
    bh[n] = h;
    ++n;
  };
  if (wR < g.pw) add(1, wR, g.ph);
  if (hB < g.ph) add(2, g.pw, hB);
  if (wR < g.pw && hB < g.ph) add(3, wR, hB);
  for (int a = 0; a < n; ++a)  // by rows descending, then kind
    for (int b = a + 1; b < n; ++b)
      if (rows[b] > rows[a] || (rows[b] == rows[a] && kind[b] < kind[a])) {
        std::swap(kind[a], kind[b]);
        std::swap(rows[a], rows[b]);
        std::swap(bw[a], bw[b]);
        std::swap(bh[a], bh[b]);
      }
  return n;
}

bsa_status launch_attn_fwd(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                           const int32_t* row_ptr, const int32_t* col_idx, int per_head,
                           float scale, void* o, float* lse, cudaStream_t st) {
  const Geometry& g = plan.g;
  // one list for every (batch, head), 128-slot blocks: two query tiles per
  // CTA share every key tile (attn_pair.cu)
  if (attn_pair_applies(g, per_head))
    return launch_attn_pair(plan, q, k, v, row_ptr, col_idx, scale, o, lse, st);
  // a list per (batch, head), 128-slot blocks: the persistent kernel of
  // attn_draft.cu, one CTA per SM over all query tiles
  if (per_head && g.block == kTile)
    return launch_attn_draft(plan, q, k, v, row_ptr, col_idx, per_head, scale, o, lse, st,
                             /*slot=*/true);
  const int64_t rows = (int64_t)g.B * g.Hh * g.Npad;
  if (rows >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "B*Hh*Npad must be < 2^31");
  const bool fine = g.block < kTile;
  if (fine && g.ntiles > kFineMaxTiles)
    return set_error(BSA_ERR_UNSUPPORTED, "blocks smaller than 128 slots need Npad <= 262144");
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, rows, g.D) || !make_tmap(&tk, k, rows, g.D) || !make_tmap(&tv, v, rows, g.D))
    return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  const AttnParams p = make_params(plan, row_ptr, col_idx, per_head, scale, o, lse);
  const dim3 grid((unsigned)g.ntiles, (unsigned)g.Hh, (unsigned)g.B);
  cudaError_t e;
  if (g.D == 128)
    e = fine ? launch_t<128, true>(tq, tk, tv, p, grid, st) : launch_t<128, false>(tq, tk, tv, p, grid, st);
  else
    e = fine ? launch_t<64, true>(tq, tk, tv, p, grid, st) : launch_t<64, false>(tq, tk, tv, p, grid, st);
  if (e != cudaSuccess) return cuda_error(e, "attention launch");
  return BSA_OK;
}

bsa_status launch_attn_fwd_natural(const bsa_plan_s& plan, const void* q, const void* k,
                                   const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                   int per_head, float scale, void* o, float* lse,
                                   cudaStream_t st) {
  // bf16 tiles: the persistent kernel of attn_draft.cu
  return launch_attn_draft(plan, q, k, v, row_ptr, col_idx, per_head, scale, o, lse, st);
}

bsa_status launch_attn_fwd_natural_e4m3(const bsa_plan_s& plan, const void* q8, const void* k8,
                                        const void* v8, const float* scales,
                                        const int32_t* row_ptr, const int32_t* col_idx,
                                        int per_head, float scale, void* o, float* lse,
                                        cudaStream_t st) {
  const Geometry& g = plan.g;
  if (g.layout != BSA_LAYOUT_TILE || g.block != kTile)
    return set_error(BSA_ERR_UNSUPPORTED,
                     "e4m3 attention needs a TILE plan with pool_h * pool_w = 128");
  if (g.D != 128) return set_error(BSA_ERR_UNSUPPORTED, "e4m3 attention supports D = 128");
  // e4m3 tiles: the persistent kernel of attn_draft.cu
  return launch_attn_draft(plan, q8, k8, v8, row_ptr, col_idx, per_head, scale, o, lse, st,
                           /*slot=*/false, scales);
}

}  // namespace bsa
