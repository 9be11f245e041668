// LVSA frame mask ("LVSA: Training-Free Sparse Attention for Long Video
// Diffusion", section 2 "Core mechanism"):
//   rotating global anchors: G_s = {f : (f - s) mod T_per == 0}, so the
//     anchor grid shifts with the denoising step s and every frame is an
//     anchor exactly once per T_per steps;
//   extended adaptive window: a window centred on the query frame t that
//     grows past the anchors it overlaps until |A(t)| = C, A(t) = G_s U W(t);
// then expanded to key blocks on the frame layout (every block of every frame
// in A(t), ascending) for each query block of frame t.
//
// Growth order.  By default a right and a left pointer take turns, right
// first, each skipping frames already present (the anchors); a side that
// runs off the grid stops and the other continues.  With base = G_s U {t},
// need = C - |base| and nR / nL frames outside base right / left of t, the
// right side then takes kR = min(nR, max(ceil(need/2), need - nL)) of its
// frames outside base, nearest first, and the left side the other
// need - kR of its own.  The other order (distance: t+1, t-1, t+2, t-2, ...,
// skipping frames outside [0, T) and frames already present) admits a frame
// f outside base iff fewer than `need` frames outside base come before it
// (closer to t, or at the same distance on the right).  Either way each
// thread decides membership for its frames in O(1) from a prefix-sum rank,
// so the set needs no serial loop.
//
// Variants (chosen by the caller): T_per = 0 means no anchors (the sliding
// window); fixed-grid anchors are the rotating ones at s = 0.
//
// One CTA per query block (grid nbf x T); each writes its CSR row.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;

// In-place exclusive prefix sum of a[0..n) by the whole CTA; returns the total.
__device__ int block_exclusive_scan(int* a, int n, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + threadIdx.x;
    const int v = i < n ? a[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      if (w < warp) before += warp_tot[w];
      total += warp_tot[w];
    }
    if (i < n) a[i] = carry + before + x - v;
    carry += total;
    __syncthreads();
  }
  return carry;
}

__global__ void __launch_bounds__(kThreads)
    lvsa_mask_kernel(int T, int C, int T_per, int s, int alternate, int nbf,
                     int32_t* __restrict__ frame_sets,
                     int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                     unsigned int* status) {
  extern __shared__ int sh[];
  int* out = sh;                // [T+1] frames outside base -> exclusive prefix
  int* incl = sh + T + 1;       // [T+1] membership of A(t)  -> exclusive prefix
  int* members = incl + T + 1;  // [C]
  __shared__ int warp_tot[kThreads / 32];
  const int i = blockIdx.x, t = blockIdx.y;
  const int sm = T_per > 0 ? ((s % T_per) + T_per) % T_per : 0;

  for (int f = threadIdx.x; f < T; f += kThreads) {
    bool anchor = false;
    if (T_per > 0) {
      int r = (f - sm) % T_per;
      if (r < 0) r += T_per;
      anchor = r == 0;
    }
    out[f] = (anchor || f == t) ? 0 : 1;
  }
  __syncthreads();
  const int n_out = block_exclusive_scan(out, T, warp_tot);
  if (threadIdx.x == 0) out[T] = n_out;
  __syncthreads();
  const int need = C - (T - n_out);

  // number of frames outside base strictly between a and b (a < b)
  auto between = [&](int a, int b) -> int {
    const int lo = max(a + 1, 0), hi = min(b, T);
    return hi > lo ? out[hi] - out[lo] : 0;
  };
  // alternating order: frames outside base right / left of t, and each side's share
  const int nR = out[T] - out[t + 1], nL = out[t];
  const int kR = min(nR, max((need + 1) / 2, need - nL)), kL = need - kR;
  for (int f = threadIdx.x; f < T; f += kThreads) {
    const bool is_out = (out[f + 1] - out[f]) != 0;
    int in = 1;
    if (is_out && alternate) {
      // rank of f among its side's frames outside base, nearest first (1-based)
      in = f > t ? (out[f + 1] - out[t + 1] <= kR) : (out[t] - out[f] <= kL);
    } else if (is_out) {
      const int d = f > t ? f - t : t - f;
      int before = between(t, t + d) + between(t - d, t);
      if (f < t && t + d < T && (out[t + d + 1] - out[t + d]) != 0) ++before;
      in = before < need;
    }
    incl[f] = in;
  }
  __syncthreads();
  const int cnt = block_exclusive_scan(incl, T, warp_tot);
  for (int f = threadIdx.x; f < T; f += kThreads) {
    const bool in = (f + 1 < T ? incl[f + 1] : cnt) - incl[f];
    if (in && incl[f] < C) members[incl[f]] = f;
  }
  if (cnt != C && threadIdx.x == 0) {
    atomicOr(status, kStatusBadBlocklist);  // cannot happen for arguments the host accepted
    for (int k = min(cnt, C); k < C; ++k) members[k] = 0;
  }
  __syncthreads();

  if (frame_sets && i == 0)
    for (int c = threadIdx.x; c < C; c += kThreads) frame_sets[(int64_t)t * C + c] = members[c];
  const int per_row = C * nbf;
  const int64_t r = (int64_t)t * nbf + i;
  int32_t* dst = col_idx + r * per_row;
  for (int e = threadIdx.x; e < per_row; e += kThreads) {
    const int fi = e / nbf;
    dst[e] = members[fi] * nbf + (e - fi * nbf);
  }
  if (threadIdx.x == 0) row_ptr[r] = (int32_t)(r * per_row);
  if (r == (int64_t)T * nbf - 1 && threadIdx.x == 0)
    row_ptr[r + 1] = (int32_t)((r + 1) * per_row);
}

}  // namespace

cudaError_t launch_lvsa_mask(const Geometry& g, int C, int T_per, int s, int alternate,
                             int32_t* frame_sets, int32_t* row_ptr, int32_t* col_idx,
                             unsigned int* status, cudaStream_t st) {
  const size_t smem = (size_t)(2 * (g.T + 1) + C) * sizeof(int);
  const dim3 grid((unsigned)g.nbf, (unsigned)g.T);
  lvsa_mask_kernel<<<grid, kThreads, smem, st>>>(g.T, C, T_per, s, alternate, g.nbf, frame_sets,
                                                  row_ptr, col_idx, status);
  return cudaGetLastError();
}

}  // namespace bsa
