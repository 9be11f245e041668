// Reorder between the natural token layout [B, N, Hh, D] and the slot layout
// [B, Hh, Npad, D] (Draft Attention article, reorder paragraph and figure
// "Full Map" vs "Reordered Full Map": scattered blocks of the sparse mask
// become contiguous so that block-sparse attention runs on dense tiles).
//
// Both directions are pure copies, bound by HBM bandwidth: each thread moves
// 16-byte vectors, consecutive threads touch consecutive 16-byte chunks of
// the output, and each input access is a whole 16-byte chunk of a contiguous
// D-element row (256 B at D = 128).  Index arithmetic uses precomputed
// magic-number division.  The forward direction writes every slot, empty
// slots as zero, so an output buffer needs no separate clearing.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct SlotMap {
  int layout;
  uint32_t H, W, P, T;
  uint32_t block_log2;      // block is a power of two (a divisor of 128)
  uint32_t ph, pw, TH, TW;
  uint32_t frame_slots;     // frame layout: nbf * block
  uint32_t nblocks;
  FastDiv div_frame_slots;  // frame layout: slot -> frame
  FastDiv div_tiles_per_frame, div_TW, div_pw, div_ph, div_W, div_P;

  // token index (within its batch) held by `slot`, or -1 for an empty slot
  __device__ __forceinline__ int32_t token_of(uint32_t slot) const {
    if (layout == BSA_LAYOUT_FRAME) {
      uint32_t t, r;
      div_frame_slots.divmod(slot, t, r);
      if (r >= P || t >= T) return -1;
      return (int32_t)(t * P + r);
    }
    const uint32_t blk = slot >> block_log2;
    if (blk >= nblocks) return -1;
    const uint32_t e = slot & ((1u << block_log2) - 1u);
    uint32_t a, b, t, rem, i, j;
    div_pw.divmod(e, a, b);
    div_tiles_per_frame.divmod(blk, t, rem);
    div_TW.divmod(rem, i, j);
    const uint32_t y = i * ph + a, x = j * pw + b;
    if (y >= H || x >= W) return -1;
    return (int32_t)((t * H + y) * W + x);
  }
  // slot of token n (within its batch)
  __device__ __forceinline__ uint32_t slot_of(uint32_t n) const {
    uint32_t t, r;
    div_P.divmod(n, t, r);
    if (layout == BSA_LAYOUT_FRAME) return t * frame_slots + r;
    uint32_t y, x, i, a, j, b;
    div_W.divmod(r, y, x);
    div_ph.divmod(y, i, a);
    div_pw.divmod(x, j, b);
    return (((t * TH + i) * TW + j) << block_log2) + a * pw + b;
  }
};

SlotMap make_map(const Geometry& g) {
  SlotMap m;
  m.layout = g.layout;
  m.H = g.H;
  m.W = g.W;
  m.P = g.P;
  m.T = g.T;
  uint32_t l = 0;
  while ((1 << l) < g.block) ++l;
  m.block_log2 = l;
  m.ph = g.ph > 0 ? g.ph : 1;
  m.pw = g.pw > 0 ? g.pw : 1;
  m.TH = g.TH;
  m.TW = g.TW;
  m.frame_slots = (uint32_t)(g.nbf * g.block);
  m.nblocks = (uint32_t)g.nblocks;
  m.div_frame_slots = FastDiv(m.frame_slots ? m.frame_slots : 1);
  m.div_tiles_per_frame = FastDiv(g.TH * g.TW > 0 ? g.TH * g.TW : 1);
  m.div_TW = FastDiv(g.TW > 0 ? g.TW : 1);
  m.div_pw = FastDiv(m.pw);
  m.div_ph = FastDiv(m.ph);
  m.div_W = FastDiv(g.W);
  m.div_P = FastDiv(g.P);
  return m;
}

struct Ptrs3 {
  const uint4* x[3];
  uint4* y[3];
};

// Output chunk idx = (bh*Npad + slot)*cpr + c, cpr = D/8 chunks per row.
// Input chunk = ((b*N + n)*Hh + h)*cpr + c.
__global__ void __launch_bounds__(kThreads)
    reorder_fwd_kernel(Ptrs3 ptr, SlotMap map, uint32_t N, uint32_t Hh, uint32_t cpr_log2,
                       uint32_t total, FastDiv div_Npad, FastDiv div_Hh, uint32_t write_pads) {
  const uint4* __restrict__ src = ptr.x[blockIdx.y];
  uint4* __restrict__ dst = ptr.y[blockIdx.y];
  const uint32_t cmask = (1u << cpr_log2) - 1u;
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t base = blockIdx.x * kThreads + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
    bool put[kUnroll];  // a token's slot, or an empty slot when pads are written
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t idx = base + u * stride;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      put[u] = false;
      if (idx < total) {
        uint32_t bh, slot, b, h;
        div_Npad.divmod(idx >> cpr_log2, bh, slot);
        div_Hh.divmod(bh, b, h);
        const int32_t n = map.token_of(slot);
        put[u] = n >= 0 || write_pads;
        if (n >= 0)
          v[u] = __ldg(src + ((((int64_t)b * N + n) * Hh + h) << cpr_log2) + (idx & cmask));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (put[u]) dst[base + u * stride] = v[u];
  }
}

// Output chunk idx = ((b*N + n)*Hh + h)*cpr + c (natural layout).
__global__ void __launch_bounds__(kThreads)
    reorder_inv_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, SlotMap map,
                       uint32_t Npad, uint32_t Hh, uint32_t cpr_log2, uint32_t total,
                       FastDiv div_Hh, FastDiv div_N) {
  const uint32_t cmask = (1u << cpr_log2) - 1u;
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t base = blockIdx.x * kThreads + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t idx = base + u * stride;
      if (idx < total) {
        uint32_t bn, h, b, n;
        div_Hh.divmod(idx >> cpr_log2, bn, h);
        div_N.divmod(bn, b, n);
        const uint32_t slot = map.slot_of(n);
        v[u] = __ldg(src + ((((int64_t)b * Hh + h) * Npad + slot) << cpr_log2) + (idx & cmask));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t idx = base + u * stride;
      if (idx < total) dst[idx] = v[u];
    }
  }
}

uint32_t log2_exact(int v) {
  uint32_t l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

unsigned grid_for(uint64_t total) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // up to 8 resident CTAs per SM, each thread kUnroll chunks per pass
  const uint64_t want = (total + (uint64_t)kThreads * kUnroll - 1) / ((uint64_t)kThreads * kUnroll);
  const uint64_t cap = (uint64_t)sms * 8;
  return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_reorder_fwd(const Geometry& g, const void* const x[3], void* const y[3], int nt,
                               bool write_pads, cudaStream_t st) {
  const SlotMap map = make_map(g);
  Ptrs3 p;
  for (int i = 0; i < 3; ++i) {
    p.x[i] = reinterpret_cast<const uint4*>(i < nt ? x[i] : x[0]);
    p.y[i] = reinterpret_cast<uint4*>(i < nt ? y[i] : y[0]);
  }
  const uint32_t cpr_log2 = log2_exact(g.D / 8);
  const uint64_t total = (uint64_t)g.B * g.Hh * g.Npad << cpr_log2;
  const dim3 grid(grid_for(total), (unsigned)nt);
  reorder_fwd_kernel<<<grid, kThreads, 0, st>>>(p, map, (uint32_t)(g.T * g.P), (uint32_t)g.Hh,
                                                cpr_log2, (uint32_t)total,
                                                FastDiv((uint32_t)g.Npad), FastDiv((uint32_t)g.Hh),
                                                write_pads ? 1u : 0u);
  return cudaGetLastError();
}

cudaError_t launch_reorder_inv(const Geometry& g, const void* x_slots, void* x_nat,
                               cudaStream_t st) {
  const SlotMap map = make_map(g);
  const uint32_t cpr_log2 = log2_exact(g.D / 8);
  const uint64_t total = (uint64_t)g.B * g.T * g.P * g.Hh << cpr_log2;
  reorder_inv_kernel<<<grid_for(total), kThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(x_slots), reinterpret_cast<uint4*>(x_nat), map,
      (uint32_t)g.Npad, (uint32_t)g.Hh, cpr_log2, (uint32_t)total, FastDiv((uint32_t)g.Hh),
      FastDiv((uint32_t)(g.T * g.P)));
  return cudaGetLastError();
}

}  // namespace bsa
