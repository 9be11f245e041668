// Internal declarations shared by the library's translation units: the plan,
// status bits, integer helpers and launch entry points of each kernel file.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "bsattn.h"

namespace bsa {

// Bits of the plan's device status word (set with atomicOr by kernels).
enum : unsigned int {
  kStatusBadBlocklist = 1u << 0,
  kStatusTimeout = 1u << 1,
};

// Division of a 32-bit unsigned n < 2^31 by an invariant divisor d >= 1 with
// one multiply-high, add and shift (Granlund & Montgomery, "Division by
// Invariant Integers using Multiplication", PLDI 1994, section 4):
// with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// q = (mulhi(m, n) + n) >> l.  The add cannot overflow because n < 2^31.
struct FastDiv {
  uint32_t d = 1, m = 0, l = 0;
  FastDiv() = default;
  explicit FastDiv(uint32_t div) : d(div) {
    l = 0;
    while ((1ull << l) < div) ++l;
    m = (uint32_t)((((1ull << l) - div) << 32) / div + 1);
  }
  __host__ __device__ __forceinline__ uint32_t div(uint32_t n) const {
#ifdef __CUDA_ARCH__
    return (__umulhi(m, n) + n) >> l;
#else
    return (uint32_t)((((uint64_t)m * n) >> 32) + n) >> l;
#endif
  }
  __host__ __device__ __forceinline__ void divmod(uint32_t n, uint32_t& q, uint32_t& r) const {
    q = div(n);
    r = n - q * d;
  }
};

// Geometry of the token <-> slot maps, passed by value to kernels.
struct Geometry {
  int B, Hh, D, T, H, W;
  int layout;           // bsa_layout
  int ph, pw, block;
  int nbf;              // frame layout: blocks per frame
  int TH, TW;           // tile layout: tiles per column / row
  int P;                // tokens per frame (H*W)
  int64_t nblocks;      // blocks per (b, head)
  int64_t Npad;         // slots per (b, head), multiple of 128
  int64_t ntiles;       // Npad / 128
};

}  // namespace bsa

struct bsa_plan_s {
  bsa::Geometry g;
  int device = 0;
  uint32_t* d_tile_valid = nullptr;  // [ntiles][4] bit per slot: slot holds a token
  unsigned int* d_status = nullptr;  // device status word
  uint64_t wait_limit_ns = 2000000000ull;
  int lvsa_anchors = BSA_ANCHORS_ROTATING;  // bsa_plan_set_lvsa_variant
  int lvsa_window = BSA_WINDOW_ALTERNATE;
  int draft_pooling = BSA_POOL_MEAN;        // bsa_plan_set_draft_pooling
  int draft_precision = BSA_DRAFT_FP64;     // bsa_plan_set_draft_precision
  int reorder_pads = BSA_PADS_WRITE;        // bsa_plan_set_reorder_pads
  uint32_t* d_amax = nullptr;               // [3][B][Hh] scratch of bsa_quantize_e4m3
};

namespace bsa {

// Records a message for bsa_last_error() and returns `st`.
bsa_status set_error(bsa_status st, const std::string& msg);
bsa_status cuda_error(cudaError_t e, const char* what);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel launchers (each in its own translation unit).
// T_per = 0: no anchors; alternate != 0: alternating window growth.
cudaError_t launch_lvsa_mask(const Geometry& g, int C, int T_per, int s, int alternate,
                             int32_t* frame_sets, int32_t* row_ptr, int32_t* col_idx,
                             unsigned int* status, cudaStream_t st);
cudaError_t launch_reorder_fwd(const Geometry& g, const void* const x[3], void* const y[3],
                               int nt, bool write_pads, cudaStream_t st);
cudaError_t launch_reorder_inv(const Geometry& g, const void* x_slots, void* x_nat,
                               cudaStream_t st);
cudaError_t launch_draft_mask(const Geometry& g, const uint32_t* tile_valid, const void* q,
                              const void* k, int keep, int pooling, int precision,
                              int32_t* row_ptr, int32_t* kv_idx, float* draft_map, void* ws,
                              cudaStream_t st, bool natural = false, uint32_t* amax = nullptr,
                              bool* amax_recorded = nullptr);

// e4m3 quantization of natural-layout Q, K, V (scales [3][B][Hh]).
// qk_amax_ready: amax_ws already holds the maxima of Q and K (and zero for V).
cudaError_t launch_quantize_e4m3(const Geometry& g, uint32_t* amax_ws, const void* q, const void* k,
                                 const void* v, void* q8, void* k8, void* v8, float* scales,
                                 cudaStream_t st, bool qk_amax_ready = false);
// Natural-layout attention on e4m3 Q, K, V (TILE plan, 128-slot tiles, D = 128).
bsa_status launch_attn_fwd_natural_e4m3(const bsa_plan_s& plan, const void* q8, const void* k8,
                                        const void* v8, const float* scales,
                                        const int32_t* row_ptr, const int32_t* col_idx,
                                        int per_head, float scale, void* o, float* lse,
                                        cudaStream_t st);

// Anchor grid actually used for (plan variant, T_per, s): *T_per_eff = 0
// means no anchors; also returns |G| over the plan's T frames.
int lvsa_effective_anchors(const bsa_plan_s* plan, int T_per, int s, int* T_per_eff, int* s_eff);
bsa_status launch_attn_fwd(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                           const int32_t* row_ptr, const int32_t* col_idx, int per_head,
                           float scale, void* o, float* lse, cudaStream_t st);
// The same on natural-layout [B, N, Hh, D] tensors for a TILE plan whose
// tiles are 128 slots (pool_h * pool_w = 128); LSE as [B, Hh, N].
bsa_status launch_attn_fwd_natural(const bsa_plan_s& plan, const void* q, const void* k,
                                   const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                   int per_head, float scale, void* o, float* lse,
                                   cudaStream_t st);
// The same, persistent (one CTA per SM over all query tiles), bf16 tiles.
// slot = true: the slot tensors [B, Hh, Npad, D] of any plan with 128-slot
// blocks instead (LSE as [B, Hh, Npad]; empty slots written as 0 / -inf).
// fp8_scales != null: natural-layout e4m3 tiles with those [3][B][Hh] scales
// (8-bit MMAs, P rounded to e4m3; D = 128).
bsa_status launch_attn_draft(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                             const int32_t* row_ptr, const int32_t* col_idx, int per_head,
                             float scale, void* o, float* lse, cudaStream_t st, bool slot = false,
                             const float* fp8_scales = nullptr);
// Shared block lists (per_head = 0) with 128-slot blocks: two query tiles per
// CTA over the union of their rows (attn_pair.cu).
bool attn_pair_applies(const Geometry& g, int per_head);
bsa_status launch_attn_pair(const bsa_plan_s& plan, const void* q, const void* k, const void* v,
                            const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                            float* lse, cudaStream_t st);
// Partial-tile kinds at a TILE grid's right edge (1), bottom edge (2) and
// corner (3), largest first, with their token rows and box width / height.
int edge_kinds(const Geometry& g, int kind[3], int rows[3], int bw[3], int bh[3]);
cudaError_t launch_selftest_timeout(unsigned int* status, uint64_t limit_ns, cudaStream_t st);

// Size bookkeeping shared by the API and the draft kernels.
size_t draft_workspace_bytes(const Geometry& g, int precision);
int draft_rows_per_cta(int64_t nblocks, int precision);

}  // namespace bsa
