// C ABI of libbsattn.so: plans, argument checking, error reporting.  Each
// entry point validates on the host, then enqueues its kernel(s) on the
// caller's stream; nothing is allocated per call.
#include <cstdio>
#include <new>
#include <string>
#include <vector>

#include "bsa_internal.cuh"
#include "ptx.cuh"

namespace bsa {

int lvsa_effective_anchors(const bsa_plan_s* plan, int T_per, int s, int* T_per_eff, int* s_eff) {
  const int T = plan->g.T;
  if (plan->lvsa_anchors == BSA_ANCHORS_NONE) {
    *T_per_eff = 0;
    *s_eff = 0;
    return 0;
  }
  *T_per_eff = T_per;
  *s_eff = plan->lvsa_anchors == BSA_ANCHORS_FIXED ? 0 : ((s % T_per) + T_per) % T_per;
  int n = 0;
  for (int f = 0; f < T; ++f) n += ((f - *s_eff) % T_per + T_per) % T_per == 0;
  return n;
}


static thread_local std::string g_last_error;

bsa_status set_error(bsa_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

bsa_status cuda_error(cudaError_t e, const char* what) {
  return set_error(BSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

namespace {

bool slot_holds_token(const Geometry& g, int64_t slot) {
  if (g.layout == BSA_LAYOUT_FRAME) {
    const int64_t fs = (int64_t)g.nbf * g.block;
    const int64_t t = slot / fs, r = slot % fs;
    return t < g.T && r < g.P;
  }
  const int64_t blk = slot / g.block;
  if (blk >= g.nblocks) return false;
  const int64_t e = slot % g.block;
  const int64_t a = e / g.pw, b = e % g.pw;
  const int64_t rem = blk % ((int64_t)g.TH * g.TW);
  const int64_t i = rem / g.TW, j = rem % g.TW;
  return i * g.ph + a < g.H && j * g.pw + b < g.W;
}

__global__ void selftest_timeout_kernel(unsigned int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx wc{status, &abort_flag, limit_ns};
  // nobody arrives on `bar`: the wait must run out and record the timeout
  bounded_wait(&bar, 0, wc);
}

bsa_status check_ptr(const void* p, const char* name) {
  if (!p) return set_error(BSA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!aligned16(p)) return set_error(BSA_ERR_ALIGNMENT, std::string(name) + " is not 16-byte aligned");
  return BSA_OK;
}

}  // namespace

cudaError_t launch_selftest_timeout(unsigned int* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace bsa

using namespace bsa;

extern "C" {

const char* bsa_last_error(void) { return g_last_error.c_str(); }

const char* bsa_version(void) { return "bsattn 0.1.0 (sm_100a)"; }

bsa_status bsa_plan_create(bsa_plan_t* plan, int B, int Hh, int D, int T, int H, int W, int layout,
                           int pool_h, int pool_w, int block) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  *plan = nullptr;
  if (B <= 0 || Hh <= 0 || T <= 0 || H <= 0 || W <= 0 || block <= 0)
    return set_error(BSA_ERR_INVALID_ARG, "sizes must be positive");
  if (D != 64 && D != 128) return set_error(BSA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (block > 128 || (128 % block) != 0)
    return set_error(BSA_ERR_UNSUPPORTED, "block must divide 128");
  Geometry g{};
  g.B = B;
  g.Hh = Hh;
  g.D = D;
  g.T = T;
  g.H = H;
  g.W = W;
  g.layout = layout;
  g.block = block;
  if ((int64_t)H * W >= (1ll << 31)) return set_error(BSA_ERR_UNSUPPORTED, "frame too large");
  g.P = H * W;
  if (layout == BSA_LAYOUT_FRAME) {
    g.ph = g.pw = 0;
    g.nbf = (g.P + block - 1) / block;
    g.TH = g.TW = 0;
    g.nblocks = (int64_t)T * g.nbf;
  } else if (layout == BSA_LAYOUT_TILE) {
    if (pool_h <= 0 || pool_w <= 0)
      return set_error(BSA_ERR_INVALID_ARG, "pool_h and pool_w must be positive");
    if ((int64_t)pool_h * pool_w != block)
      return set_error(BSA_ERR_INVALID_ARG, "pool_h * pool_w must equal the block size");
    g.ph = pool_h;
    g.pw = pool_w;
    g.TH = (H + pool_h - 1) / pool_h;
    g.TW = (W + pool_w - 1) / pool_w;
    g.nbf = g.TH * g.TW;
    g.nblocks = (int64_t)T * g.TH * g.TW;
  } else {
    return set_error(BSA_ERR_INVALID_ARG, "unknown layout");
  }
  g.Npad = (g.nblocks * block + 127) / 128 * 128;
  g.ntiles = g.Npad / 128;
  const int64_t chunks = (int64_t)B * Hh * g.Npad * (D / 8);
  const int64_t nat_chunks = (int64_t)B * T * g.P * Hh * (D / 8);
  if (chunks >= (1ll << 31) || nat_chunks >= (1ll << 31) || g.nblocks >= (1ll << 30))
    return set_error(BSA_ERR_UNSUPPORTED, "problem too large (index range)");

  // no exception may cross the C ABI: host allocations are checked here
  std::vector<uint32_t> tv;
  try {
    tv.assign((size_t)g.ntiles * 4, 0u);
  } catch (const std::bad_alloc&) {
    return set_error(BSA_ERR_INVALID_ARG, "host memory for the slot map");
  }
  for (int64_t s = 0; s < g.Npad; ++s)
    if (slot_holds_token(g, s)) tv[(size_t)(s >> 5)] |= 1u << (s & 31);

  auto* p = new (std::nothrow) bsa_plan_s;
  if (!p) return set_error(BSA_ERR_INVALID_ARG, "host memory for the plan");
  p->g = g;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaMalloc(&p->d_tile_valid, tv.size() * sizeof(uint32_t));
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_tile_valid, tv.data(), tv.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMalloc(&p->d_status, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMalloc(&p->d_amax, sizeof(uint32_t) * 3 * B * Hh);
  if (e != cudaSuccess) {
    if (p->d_tile_valid) cudaFree(p->d_tile_valid);
    if (p->d_status) cudaFree(p->d_status);
    if (p->d_amax) cudaFree(p->d_amax);
    delete p;
    return cuda_error(e, "plan allocation");
  }
  *plan = p;
  return BSA_OK;
}

bsa_status bsa_plan_destroy(bsa_plan_t plan) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(plan->device);
  cudaFree(plan->d_tile_valid);
  cudaFree(plan->d_status);
  cudaFree(plan->d_amax);
  cudaSetDevice(cur);
  delete plan;
  return BSA_OK;
}

int64_t bsa_padded_tokens(bsa_plan_t plan) { return plan ? plan->g.Npad : -1; }
int64_t bsa_num_blocks(bsa_plan_t plan) { return plan ? plan->g.nblocks : -1; }
int bsa_block_size(bsa_plan_t plan) { return plan ? plan->g.block : -1; }

int64_t bsa_lvsa_nnz(bsa_plan_t plan, int C) {
  if (!plan || plan->g.layout != BSA_LAYOUT_FRAME || C <= 0) return -1;
  return plan->g.nblocks * (int64_t)C * plan->g.nbf;
}

bsa_status bsa_lvsa_mask(bsa_plan_t plan, int C, int T_per, int s, int32_t* frame_sets,
                         int32_t* row_ptr, int32_t* col_idx, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_FRAME) return set_error(BSA_ERR_INVALID_ARG, "LVSA mask needs a FRAME plan");
  if (T_per < 1) return set_error(BSA_ERR_INVALID_ARG, "T_per must be >= 1");
  if (C < 1 || C > g.T) return set_error(BSA_ERR_INVALID_ARG, "C must be in [1, T]");
  if (!row_ptr || !col_idx) return set_error(BSA_ERR_INVALID_ARG, "row_ptr / col_idx is NULL");
  if ((int64_t)g.nblocks * C * g.nbf >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  // |G U {t}| <= C for every t
  int tp = 0, sm = 0;
  const int anchors = lvsa_effective_anchors(plan, T_per, s, &tp, &sm);
  const int worst = anchors + (anchors < g.T ? 1 : 0);
  if (worst > C)
    return set_error(BSA_ERR_INVALID_ARG, "budget C is smaller than the anchors plus the query frame");
  cudaError_t e = launch_lvsa_mask(g, C, tp, sm, plan->lvsa_window == BSA_WINDOW_ALTERNATE,
                                   frame_sets, row_ptr, col_idx, plan->d_status,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "lvsa_mask launch");
}

int bsa_draft_keep_count(bsa_plan_t plan, int sparsity_pct) {
  if (!plan || sparsity_pct < 0 || sparsity_pct >= 100) return -1;
  const int64_t nb = plan->g.nblocks;
  return (int)((nb * (100 - sparsity_pct) + 99) / 100);
}

size_t bsa_draft_workspace_bytes(bsa_plan_t plan) {
  return plan ? draft_workspace_bytes(plan->g, plan->draft_precision) : 0;
}

bsa_status bsa_draft_mask(bsa_plan_t plan, const void* q_slots, const void* k_slots,
                          int sparsity_pct, int32_t* row_ptr, int32_t* kv_idx, float* draft_map,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_TILE) return set_error(BSA_ERR_INVALID_ARG, "draft mask needs a TILE plan");
  if (sparsity_pct < 0 || sparsity_pct >= 100)
    return set_error(BSA_ERR_INVALID_ARG, "sparsity must be in [0, 100)");
  bsa_status st;
  if ((st = check_ptr(q_slots, "q_slots")) != BSA_OK) return st;
  if ((st = check_ptr(k_slots, "k_slots")) != BSA_OK) return st;
  if ((st = check_ptr(workspace, "workspace")) != BSA_OK) return st;
  if (!kv_idx) return set_error(BSA_ERR_INVALID_ARG, "kv_idx is NULL");
  if (workspace_bytes < draft_workspace_bytes(g, plan->draft_precision))
    return set_error(BSA_ERR_INVALID_ARG, "workspace too small");
  if (g.nblocks > 18000) return set_error(BSA_ERR_UNSUPPORTED, "draft mask supports up to 18000 blocks");
  if ((int64_t)g.B * g.Hh * g.Npad >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "draft mask needs B*Hh*Npad < 2^31");
  const int keep = bsa_draft_keep_count(plan, sparsity_pct);
  if ((int64_t)g.B * g.Hh * g.nblocks * keep >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  cudaError_t e = launch_draft_mask(g, plan->d_tile_valid, q_slots, k_slots, keep,
                                    plan->draft_pooling, plan->draft_precision, row_ptr, kv_idx,
                                    draft_map, workspace, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask launch");
}

bsa_status bsa_reorder_fwd(bsa_plan_t plan, const void* x0, void* y0, const void* x1, void* y1,
                           const void* x2, void* y2, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  bsa_status st;
  if ((st = check_ptr(x0, "x0")) != BSA_OK || (st = check_ptr(y0, "y0")) != BSA_OK) return st;
  const void* xs[3] = {x0, x1, x2};
  void* ys[3] = {y0, y1, y2};
  // pairs 1 and 2 are optional, in order: a pair after an absent one is an error
  int nt = 1;
  for (int i = 1; i < 3; ++i) {
    if (!xs[i] && !ys[i]) break;
    if ((st = check_ptr(xs[i], "x")) != BSA_OK || (st = check_ptr(ys[i], "y")) != BSA_OK) return st;
    nt = i + 1;
  }
  for (int i = nt + 1; i < 3; ++i)
    if (xs[i] || ys[i])
      return set_error(BSA_ERR_INVALID_ARG, "tensor pair 2 given without pair 1");
  cudaError_t e = launch_reorder_fwd(plan->g, xs, ys, nt, plan->reorder_pads == BSA_PADS_WRITE,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "reorder_fwd launch");
}

bsa_status bsa_reorder_inv(bsa_plan_t plan, const void* x_slots, void* x_nat, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  bsa_status st;
  if ((st = check_ptr(x_slots, "x_slots")) != BSA_OK || (st = check_ptr(x_nat, "x_nat")) != BSA_OK)
    return st;
  cudaError_t e = launch_reorder_inv(plan->g, x_slots, x_nat, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "reorder_inv launch");
}

bsa_status bsa_attn_fwd(bsa_plan_t plan, const void* q, const void* k, const void* v,
                        const int32_t* row_ptr, const int32_t* col_idx, int per_head_lists,
                        float scale, void* o, float* lse, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  bsa_status st;
  if ((st = check_ptr(q, "q")) != BSA_OK || (st = check_ptr(k, "k")) != BSA_OK ||
      (st = check_ptr(v, "v")) != BSA_OK || (st = check_ptr(o, "o")) != BSA_OK)
    return st;
  if (!row_ptr || !col_idx) return set_error(BSA_ERR_INVALID_ARG, "row_ptr / col_idx is NULL");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "lse is not 4-byte aligned");
  if (!(scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be positive");
  return launch_attn_fwd(*plan, q, k, v, row_ptr, col_idx, per_head_lists, scale, o, lse,
                         reinterpret_cast<cudaStream_t>(stream));
}

bsa_status bsa_attn_fwd_natural(bsa_plan_t plan, const void* q, const void* k, const void* v,
                                const int32_t* row_ptr, const int32_t* col_idx, int per_head_lists,
                                float scale, void* o, float* lse, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (plan->g.layout != BSA_LAYOUT_TILE)
    return set_error(BSA_ERR_INVALID_ARG, "natural-layout attention needs a TILE plan");
  bsa_status st;
  if ((st = check_ptr(q, "q")) != BSA_OK || (st = check_ptr(k, "k")) != BSA_OK ||
      (st = check_ptr(v, "v")) != BSA_OK || (st = check_ptr(o, "o")) != BSA_OK)
    return st;
  if (!row_ptr || !col_idx) return set_error(BSA_ERR_INVALID_ARG, "row_ptr / col_idx is NULL");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "lse is not 4-byte aligned");
  if (!(scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be positive");
  return launch_attn_fwd_natural(*plan, q, k, v, row_ptr, col_idx, per_head_lists, scale, o, lse,
                                 reinterpret_cast<cudaStream_t>(stream));
}

bsa_status bsa_draft_mask_natural(bsa_plan_t plan, const void* q, const void* k, int sparsity_pct,
                                  int32_t* row_ptr, int32_t* kv_idx, float* draft_map,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_TILE) return set_error(BSA_ERR_INVALID_ARG, "draft mask needs a TILE plan");
  if (sparsity_pct < 0 || sparsity_pct >= 100)
    return set_error(BSA_ERR_INVALID_ARG, "sparsity must be in [0, 100)");
  bsa_status st;
  if ((st = check_ptr(q, "q")) != BSA_OK) return st;
  if ((st = check_ptr(k, "k")) != BSA_OK) return st;
  if ((st = check_ptr(workspace, "workspace")) != BSA_OK) return st;
  if (!kv_idx) return set_error(BSA_ERR_INVALID_ARG, "kv_idx is NULL");
  if (workspace_bytes < draft_workspace_bytes(g, plan->draft_precision))
    return set_error(BSA_ERR_INVALID_ARG, "workspace too small");
  if (g.nblocks > 18000) return set_error(BSA_ERR_UNSUPPORTED, "draft mask supports up to 18000 blocks");
  if ((int64_t)g.B * g.Hh * g.Npad >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "draft mask needs B*Hh*Npad < 2^31");
  const int keep = bsa_draft_keep_count(plan, sparsity_pct);
  if ((int64_t)g.B * g.Hh * g.nblocks * keep >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  cudaError_t e = launch_draft_mask(g, plan->d_tile_valid, q, k, keep, plan->draft_pooling,
                                    plan->draft_precision, row_ptr, kv_idx, draft_map, workspace,
                                    reinterpret_cast<cudaStream_t>(stream), /*natural=*/true);
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "draft_mask_natural launch");
}

bsa_status bsa_draft_mask_natural_e4m3(bsa_plan_t plan, const void* q, const void* k, const void* v,
                                       int sparsity_pct, int32_t* row_ptr, int32_t* kv_idx,
                                       float* draft_map, void* workspace, size_t workspace_bytes,
                                       void* q8, void* k8, void* v8, float* scales, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  const Geometry& g = plan->g;
  if (g.layout != BSA_LAYOUT_TILE) return set_error(BSA_ERR_INVALID_ARG, "draft mask needs a TILE plan");
  if (sparsity_pct < 0 || sparsity_pct >= 100)
    return set_error(BSA_ERR_INVALID_ARG, "sparsity must be in [0, 100)");
  bsa_status st;
  if ((st = check_ptr(q, "q")) != BSA_OK || (st = check_ptr(k, "k")) != BSA_OK ||
      (st = check_ptr(v, "v")) != BSA_OK || (st = check_ptr(q8, "q8")) != BSA_OK ||
      (st = check_ptr(k8, "k8")) != BSA_OK || (st = check_ptr(v8, "v8")) != BSA_OK ||
      (st = check_ptr(workspace, "workspace")) != BSA_OK)
    return st;
  if (!scales || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "scales is NULL or not 4-byte aligned");
  if (!kv_idx) return set_error(BSA_ERR_INVALID_ARG, "kv_idx is NULL");
  if (workspace_bytes < draft_workspace_bytes(g, plan->draft_precision))
    return set_error(BSA_ERR_INVALID_ARG, "workspace too small");
  if (g.nblocks > 18000) return set_error(BSA_ERR_UNSUPPORTED, "draft mask supports up to 18000 blocks");
  if ((int64_t)g.B * g.Hh * g.Npad >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "draft mask needs B*Hh*Npad < 2^31");
  const int keep = bsa_draft_keep_count(plan, sparsity_pct);
  if ((int64_t)g.B * g.Hh * g.nblocks * keep >= (1ll << 31))
    return set_error(BSA_ERR_UNSUPPORTED, "block list longer than 2^31 entries");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the pooling reads Q and K once for the draft map and records their
  // per-(batch, head) maxima on the way; the quantization then takes only V's
  cudaError_t e = cudaMemsetAsync(plan->d_amax, 0, sizeof(uint32_t) * 3 * g.B * g.Hh, s);
  if (e != cudaSuccess) return cuda_error(e, "amax reset");
  bool recorded = false;
  e = launch_draft_mask(g, plan->d_tile_valid, q, k, keep, plan->draft_pooling,
                        plan->draft_precision, row_ptr, kv_idx, draft_map, workspace, s,
                        /*natural=*/true, plan->d_amax, &recorded);
  if (e != cudaSuccess) return cuda_error(e, "draft_mask_natural_e4m3 launch");
  e = launch_quantize_e4m3(g, plan->d_amax, q, k, v, q8, k8, v8, scales, s, recorded);
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "quantize_e4m3 launch");
}

bsa_status bsa_quantize_e4m3(bsa_plan_t plan, const void* q, const void* k, const void* v, void* q8,
                             void* k8, void* v8, float* scales, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  bsa_status st;
  if ((st = check_ptr(q, "q")) != BSA_OK || (st = check_ptr(k, "k")) != BSA_OK ||
      (st = check_ptr(v, "v")) != BSA_OK || (st = check_ptr(q8, "q8")) != BSA_OK ||
      (st = check_ptr(k8, "k8")) != BSA_OK || (st = check_ptr(v8, "v8")) != BSA_OK)
    return st;
  if (!scales || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "scales is NULL or not 4-byte aligned");
  cudaError_t e = launch_quantize_e4m3(plan->g, plan->d_amax, q, k, v, q8, k8, v8, scales,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "quantize_e4m3 launch");
}

bsa_status bsa_attn_fwd_natural_e4m3(bsa_plan_t plan, const void* q8, const void* k8,
                                     const void* v8, const float* scales, const int32_t* row_ptr,
                                     const int32_t* col_idx, int per_head_lists, float scale,
                                     void* o, float* lse, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (plan->g.layout != BSA_LAYOUT_TILE)
    return set_error(BSA_ERR_INVALID_ARG, "e4m3 attention needs a TILE plan");
  bsa_status st;
  if ((st = check_ptr(q8, "q8")) != BSA_OK || (st = check_ptr(k8, "k8")) != BSA_OK ||
      (st = check_ptr(v8, "v8")) != BSA_OK || (st = check_ptr(o, "o")) != BSA_OK)
    return st;
  if (!scales || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "scales is NULL or not 4-byte aligned");
  if (!row_ptr || !col_idx) return set_error(BSA_ERR_INVALID_ARG, "row_ptr / col_idx is NULL");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return set_error(BSA_ERR_ALIGNMENT, "lse is not 4-byte aligned");
  if (!(scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be positive");
  return launch_attn_fwd_natural_e4m3(*plan, q8, k8, v8, scales, row_ptr, col_idx, per_head_lists,
                                      scale, o, lse, reinterpret_cast<cudaStream_t>(stream));
}

bsa_status bsa_poll_status(bsa_plan_t plan, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int h = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&h, plan->d_status, sizeof(h), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(plan->d_status, 0, sizeof(h));
  if (e != cudaSuccess) return cuda_error(e, "poll_status");
  if (h & kStatusTimeout) return set_error(BSA_ERR_TIMEOUT, "a bounded device wait ran out");
  if (h & kStatusBadBlocklist)
    return set_error(BSA_ERR_BAD_BLOCKLIST, "a block list named a block out of range or was not ordered");
  return BSA_OK;
}

bsa_status bsa_plan_set_lvsa_variant(bsa_plan_t plan, int anchors, int window_order) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (anchors < BSA_ANCHORS_ROTATING || anchors > BSA_ANCHORS_NONE)
    return set_error(BSA_ERR_INVALID_ARG, "unknown anchor mode");
  if (window_order != BSA_WINDOW_DISTANCE && window_order != BSA_WINDOW_ALTERNATE)
    return set_error(BSA_ERR_INVALID_ARG, "unknown window order");
  plan->lvsa_anchors = anchors;
  plan->lvsa_window = window_order;
  return BSA_OK;
}

bsa_status bsa_plan_set_draft_pooling(bsa_plan_t plan, int pooling) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (pooling != BSA_POOL_MEAN && pooling != BSA_POOL_MAX)
    return set_error(BSA_ERR_INVALID_ARG, "unknown pooling");
  plan->draft_pooling = pooling;
  return BSA_OK;
}

bsa_status bsa_plan_set_reorder_pads(bsa_plan_t plan, int pads) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (pads != BSA_PADS_WRITE && pads != BSA_PADS_KEEP)
    return set_error(BSA_ERR_INVALID_ARG, "unknown pad mode");
  plan->reorder_pads = pads;
  return BSA_OK;
}

bsa_status bsa_plan_set_draft_precision(bsa_plan_t plan, int precision) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (precision != BSA_DRAFT_FP64 && precision != BSA_DRAFT_FP32)
    return set_error(BSA_ERR_INVALID_ARG, "unknown draft precision");
  plan->draft_precision = precision;
  return BSA_OK;
}

bsa_status bsa_set_wait_limit_ns(bsa_plan_t plan, uint64_t ns) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (ns == 0) return set_error(BSA_ERR_INVALID_ARG, "limit must be positive");
  plan->wait_limit_ns = ns;
  return BSA_OK;
}

bsa_status bsa_selftest_timeout(bsa_plan_t plan, uint64_t limit_ns, void* stream) {
  if (!plan) return set_error(BSA_ERR_INVALID_ARG, "plan is NULL");
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return set_error(BSA_ERR_INVALID_ARG, "limit must be in (0, 10 s]");
  cudaError_t e = launch_selftest_timeout(plan->d_status, limit_ns,
                                          reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BSA_OK : cuda_error(e, "selftest launch");
}

}  // extern "C"
