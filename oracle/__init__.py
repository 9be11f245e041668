"""CPU fp64 oracle for block-sparse attention over [t,h,w] video tokens.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
CPU-baseline leg of the benchmark may import this module; the product path
(the CUDA library and its Python binding) never does, and this module never
imports the product.  It is a plain, slow, obviously-correct restatement of
what the method computes, written from the pages:

* "LVSA: Training-Free Sparse Attention for Long Video Diffusion" (gist.science
  summary), section 2 "Methodology", "Core mechanism": the attended frame set
  A(t) = G_s U W(t) with rotating global anchors and an extended adaptive
  window, budget |A(t)| = C; "Complexity": T*C*P^2*d total work.
* The Draft Attention article ("科学家提出视频扩散模型加速方法，在H100实现一倍以上
  端到端加速", 163.com): tokens reshaped to [t,h,w], average-pooled Q and K give
  a low-resolution draft attention map, which yields a sparse mask that guides
  full-resolution block-sparse attention; pool_h x pool_w = block_size; a
  reorder makes the selected blocks contiguous; quantization is named as the
  next step.

All floating point is fp64 (bf16 inputs convert to fp64 exactly), except
where a float decides an integer in the kernel's precision: the e4m3 scales
and divisions are fp32, and so are the draft logits of the library's
optional fp32 draft precision (draft_logits(..., precision="fp32")).

Readings of points the pages leave open:
* window extension order: a right and a left pointer take turns, right
  first, each moving past frames already in the set (anchors) and stopping
  at the grid's edge, until |A(t)| = C (reading B, the default: the tiny
  workload's definition says the window is extended alternately right then
  left, skipping anchors, clamped at the edges); reading A, offsets +1, -1,
  +2, -2, ... around t, is available as order="distance";
* anchors G_s = {f : (f - s) mod T_per == 0}; the fixed-grid and window-only
  variants take {f : f mod T_per == 0} and the empty set;
* draft pooling averages the valid tokens of a tile only (grid-edge tiles are
  partially filled); sums run sequentially in row-major (a, then b) order and
  the mean is one IEEE division; max pooling takes the maximum over the same
  tokens;
* draft logits are a sequential multiply-then-add chain over the channels,
  each operation rounded to fp64 (no fused multiply-add); the optional fp32
  precision rounds the pooled values once to fp32 and every operation to
  fp32 (the pages fix no precision for the draft map);
* top-k per query-block row keeps k = ceil(Nb*(100-p)/100) blocks ranked by
  (logit descending, block index ascending), returned in ascending order;
* a query with no allowed valid key gets O = 0 and LSE = -inf; pad query
  slots likewise;
* fp8 (quantization, the Draft article's next step): e4m3 values, one scale
  per (batch, head) and tensor, scale = fp32(amax)/448, x/scale in fp32
  rounded to nearest even and saturated at +-448.

Parity status: every function here is pinned by tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

# ---------------------------------------------------------------------------
# LVSA frame sets  (LVSA, section 2 "Core mechanism")
# ---------------------------------------------------------------------------


ANCHOR_MODES = ("rotating", "fixed", "none")
WINDOW_ORDERS = ("alternate", "distance")


def lvsa_anchors(T: int, T_per: int, s: int, anchors: str = "rotating") -> list[int]:
    """Global anchor frames at denoising step s.

    "rotating" (LVSA, section 2, "Rotating global anchors"): the grid of
    period T_per is shifted by s mod T_per, so over T_per consecutive steps
    every frame is an anchor exactly once.  "fixed": the fixed-grid global
    frames the same section contrasts it with, {f : f mod T_per == 0} at every
    step.  "none": no global frames, the sliding-window pattern the page's
    introduction lists among earlier approaches.
    """
    if anchors == "rotating":
        return [f for f in range(T) if (f - s) % T_per == 0]
    if anchors == "fixed":
        return [f for f in range(T) if f % T_per == 0]
    if anchors == "none":
        return []
    raise ValueError(f"unknown anchor mode {anchors!r}")


def lvsa_frame_set(t: int, T: int, C: int, T_per: int, s: int, anchors: str = "rotating",
                   order: str = "alternate") -> list[int]:
    """A(t) = G_s U W(t) for query frame t, with |A(t)| = C exactly.

    W(t) is a local window centred on t that grows past anchors it overlaps so
    that the budget C is always met (LVSA, section 2, "Extended adaptive
    window").  The page does not fix the growth order; two readings:

    * "alternate" (the default): a right pointer and a left pointer take
      turns, right first; each turn moves its pointer past frames already in
      the set and adds the next frame on its side; a side that runs off the
      grid stops and the other side continues;
    * "distance": t+1, t-1, t+2, t-2, ...; frames outside [0, T) and frames
      already in the set are skipped and cost no budget.
    """
    if not (0 <= t < T) or C > T or (anchors != "none" and T_per <= 0):
        raise ValueError("bad LVSA arguments")
    if order not in WINDOW_ORDERS:
        raise ValueError(f"unknown window order {order!r}")
    A = set(lvsa_anchors(T, T_per, s, anchors))
    A.add(t)
    if len(A) > C:
        raise ValueError("budget C smaller than anchors + own frame")
    if order == "distance":
        d = 1
        while len(A) < C:
            for f in (t + d, t - d):
                if len(A) < C and 0 <= f < T and f not in A:
                    A.add(f)
            d += 1
    else:
        r, l = t + 1, t - 1
        while len(A) < C:
            while r < T and r in A:
                r += 1
            if r < T:
                A.add(r)
                r += 1
            if len(A) == C:
                break
            while l >= 0 and l in A:
                l -= 1
            if l >= 0:
                A.add(l)
                l -= 1
    return sorted(A)


def lvsa_frame_sets(T: int, C: int, T_per: int, s: int, anchors: str = "rotating",
                    order: str = "alternate") -> np.ndarray:
    """int32 [T, C]: row t is A(t) in ascending order."""
    return np.array([lvsa_frame_set(t, T, C, T_per, s, anchors, order) for t in range(T)],
                    dtype=np.int32).reshape(T, C)


# ---------------------------------------------------------------------------
# Token -> slot maps (Draft Attention article, "reorder" paragraph and figure
# "Full Map" vs "Reordered Full Map")
# ---------------------------------------------------------------------------


def frame_layout_perm(T: int, H: int, W: int, block: int):
    """Frame layout: each frame padded to whole `block`-token blocks.

    Token (t, y, x) goes to slot t*nbf*block + y*W + x, nbf = ceil(H*W/block).
    Returns (perm int64[N] natural->slot, Npad).
    """
    P = H * W
    nbf = -(-P // block)
    perm = np.empty(T * P, dtype=np.int64)
    for t in range(T):
        for y in range(H):
            for x in range(W):
                perm[(t * H + y) * W + x] = t * nbf * block + y * W + x
    return perm, T * nbf * block


def tile_layout_perm(T: int, H: int, W: int, ph: int, pw: int):
    """Tile layout: each ph x pw spatial tile of a frame is one contiguous block.

    Token (t, i*ph+a, j*pw+b) goes to slot ((t*TH + i)*TW + j)*(ph*pw) + a*pw + b
    with TH = ceil(H/ph), TW = ceil(W/pw); tiles hanging over the grid edge
    keep empty slots.  Returns (perm int64[N], Npad).
    """
    TH, TW = -(-H // ph), -(-W // pw)
    perm = np.empty(T * H * W, dtype=np.int64)
    for t in range(T):
        for y in range(H):
            for x in range(W):
                i, a = divmod(y, ph)
                j, b = divmod(x, pw)
                perm[(t * H + y) * W + x] = ((t * TH + i) * TW + j) * (ph * pw) + a * pw + b
    return perm, T * TH * TW * ph * pw


def slot_valid(perm: np.ndarray, Npad: int) -> np.ndarray:
    """bool[Npad]: True where a slot holds a real token."""
    v = np.zeros(Npad, dtype=bool)
    v[perm] = True
    return v


def reorder_fwd(x_nat: np.ndarray, perm: np.ndarray, Npad: int) -> np.ndarray:
    """[B, N, Hh, D] natural -> [B, Hh, Npad, D] slots; empty slots are zero."""
    B, N, Hh, D = x_nat.shape
    out = np.zeros((B, Hh, Npad, D), dtype=x_nat.dtype)
    out[:, :, perm, :] = np.transpose(x_nat, (0, 2, 1, 3))
    return out


def reorder_inv(x_slots: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """[B, Hh, Npad, D] slots -> [B, N, Hh, D] natural (empty slots dropped)."""
    return np.ascontiguousarray(np.transpose(x_slots[:, :, perm, :], (0, 2, 1, 3)))


# ---------------------------------------------------------------------------
# Block lists
# ---------------------------------------------------------------------------


def lvsa_block_csr(sets: np.ndarray, nbf: int):
    """Expand frame sets to a block CSR on the frame layout.

    Query block qb lies in frame t = qb // nbf and may attend every block of
    every frame in A(t), ascending (LVSA, section 2: block-sparse attention
    restricted to the frame set).  Returns (row_ptr int32[T*nbf+1], col_idx).
    """
    T = sets.shape[0]
    rows = []
    for t in range(T):
        cols = [f * nbf + i for f in sets[t] for i in range(nbf)]
        for _ in range(nbf):
            rows.append(cols)
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int64)
    for r, c in enumerate(rows):
        row_ptr[r + 1] = row_ptr[r] + len(c)
    col_idx = np.array([c for r in rows for c in r], dtype=np.int32)
    return row_ptr.astype(np.int32), col_idx


def dense_block_csr(nblocks: int):
    """Every query block attends every key block (the full mask)."""
    row_ptr = np.arange(nblocks + 1, dtype=np.int64) * nblocks
    col_idx = np.tile(np.arange(nblocks, dtype=np.int32), nblocks)
    return row_ptr.astype(np.int32), col_idx


# ---------------------------------------------------------------------------
# Draft mask (Draft Attention article: reshape to [t,h,w], average pooling,
# low-resolution attention map, sparse mask keeping the important blocks;
# pool_h x pool_w = block_size)
# ---------------------------------------------------------------------------


def draft_keep_count(Nb: int, sparsity_pct: int) -> int:
    """Blocks kept per row at `sparsity_pct` percent sparsity, never sparser."""
    if not (0 <= sparsity_pct < 100):
        raise ValueError("sparsity must be in [0, 100)")
    return (Nb * (100 - sparsity_pct) + 99) // 100


def draft_pool(x_nat: np.ndarray, T: int, H: int, W: int, ph: int, pw: int,
               mode: str = "mean") -> np.ndarray:
    """Pooling of Q or K over ph x pw tiles of each frame.

    "mean" (the article's average pooling): only tokens inside the grid
    count; the sum runs over them in row-major (a, then b) order and is
    divided once by their count.  "max" (the max pooling the article's
    authors tried first, before preferring the average at high sparsity):
    the channel-wise maximum over the same tokens, exact in any order.

    x_nat: [B, N, Hh, D] (any float dtype; converted exactly to fp64).
    Returns fp64 [B, Hh, Nb, D], Nb = T*ceil(H/ph)*ceil(W/pw), block index
    (t*TH + i)*TW + j.
    """
    if mode not in ("mean", "max"):
        raise ValueError(f"unknown pooling {mode!r}")
    B, N, Hh, D = x_nat.shape
    TH, TW = -(-H // ph), -(-W // pw)
    x = np.asarray(x_nat, dtype=np.float64).reshape(B, T, H, W, Hh, D)
    init = 0.0 if mode == "mean" else -np.inf
    acc = np.full((B, T, TH, TW, Hh, D), init, dtype=np.float64)
    cnt = np.zeros((TH, TW), dtype=np.int64)
    for a in range(ph):
        for b in range(pw):
            for i in range(TH):
                y = i * ph + a
                if y >= H:
                    continue
                for j in range(TW):
                    xx = j * pw + b
                    if xx >= W:
                        continue
                    if mode == "mean":
                        acc[:, :, i, j] = acc[:, :, i, j] + x[:, :, y, xx]
                    else:
                        acc[:, :, i, j] = np.maximum(acc[:, :, i, j], x[:, :, y, xx])
                    cnt[i, j] += 1
    pooled = acc / cnt[None, None, :, :, None, None].astype(np.float64) if mode == "mean" else acc
    # [B, T, TH, TW, Hh, D] -> [B, Hh, Nb, D]
    return np.ascontiguousarray(
        np.transpose(pooled, (0, 4, 1, 2, 3, 5)).reshape(B, Hh, T * TH * TW, D))


def draft_logits(qbar: np.ndarray, kbar: np.ndarray, precision: str = "fp64") -> np.ndarray:
    """Low-resolution logits L[b,h,i,j] = <qbar_i, kbar_j>.

    Sequential over channels c = 0..D-1: acc = acc + qbar[i,c]*kbar[j,c],
    the product and the sum each rounded (no fused multiply-add), starting
    from acc = 0.
    precision "fp64" (default): everything in fp64.
    precision "fp32": the pooled values are first rounded to fp32 (nearest,
    ties to even), and every product and sum is rounded to fp32; numpy's
    float32 multiply and add are single IEEE operations.  Returns float32.
    """
    if precision not in ("fp64", "fp32"):
        raise ValueError(f"unknown precision {precision!r}")
    dt = np.float64 if precision == "fp64" else np.float32
    qv = np.asarray(qbar, dtype=dt)
    kv = np.asarray(kbar, dtype=dt)
    B, Hh, Nb, D = qv.shape
    acc = np.zeros((B, Hh, Nb, kv.shape[2]), dtype=dt)
    for c in range(D):
        prod = qv[:, :, :, c][..., :, None] * kv[:, :, :, c][..., None, :]
        acc = acc + prod
    return acc


def draft_map(logits: np.ndarray, D: int) -> np.ndarray:
    """The draft attention map softmax(L / sqrt(D)) over key blocks (fp64)."""
    z = np.asarray(logits, dtype=np.float64) / math.sqrt(D)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def draft_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Keep the k most important key blocks of every query-block row.

    Rank by logit descending, ties to the lower block index; softmax and the
    positive 1/sqrt(D) scale are monotone per row, so ranking the logits ranks
    the draft map.  Returns int32 [..., Nq, k] ascending.
    """
    *lead, Nq, Nk = logits.shape
    flat = logits.reshape(-1, Nk)
    out = np.empty((flat.shape[0], k), dtype=np.int32)
    idx = np.arange(Nk)
    for r in range(flat.shape[0]):
        order = np.lexsort((idx, -flat[r]))
        out[r] = np.sort(order[:k])
    return out.reshape(*lead, Nq, k)


def draft_blocks(q_nat, k_nat, T, H, W, ph, pw, sparsity_pct, mode: str = "mean",
                 precision: str = "fp64"):
    """Full draft-mask pipeline: pool -> logits -> top-k.  int32 [B,Hh,Nb,k]."""
    qbar = draft_pool(q_nat, T, H, W, ph, pw, mode)
    kbar = draft_pool(k_nat, T, H, W, ph, pw, mode)
    L = draft_logits(qbar, kbar, precision)
    return draft_topk(L, draft_keep_count(L.shape[-1], sparsity_pct))


def fixed_k_csr(kv_idx: np.ndarray):
    """Per-(b,head) fixed-k lists [B,Hh,Nb,k] -> one CSR over all B*Hh*Nb rows."""
    k = kv_idx.shape[-1]
    rows = int(np.prod(kv_idx.shape[:-1]))
    row_ptr = (np.arange(rows + 1, dtype=np.int64) * k).astype(np.int32)
    return row_ptr, kv_idx.reshape(-1).astype(np.int32)


# ---------------------------------------------------------------------------
# Block-sparse softmax attention (Draft Attention article: sparse mask guides
# the full-resolution attention; LVSA section 2: block-sparse attention over
# A(t)).  Plain definition: for each valid query, softmax over the allowed
# valid keys, weighted sum of their values.
# ---------------------------------------------------------------------------


def masked_attention(q, k, v, valid: np.ndarray, block: int, row_ptr, col_idx,
                     per_head: bool, scale: float,
                     q_blocks: Optional[Sequence[int]] = None,
                     heads: Optional[Iterable[tuple]] = None):
    """Reference block-sparse attention on the slot layout.

    q, k, v: [B, Hh, Npad, D] (any float dtype; used as fp64).
    valid: bool[Npad].  Query block qb covers slots [qb*block, (qb+1)*block);
    its allowed key blocks are col_idx[row_ptr[r]:row_ptr[r+1]] with
    r = list*Nqb + qb, list = b*Hh + h if per_head else 0.
    Returns (O fp64 [B,Hh,Npad,D], LSE fp64 [B,Hh,Npad]); only the rows of
    the requested query blocks (default all) are filled, other rows are NaN.
    Pad query slots and queries with no allowed valid key get O=0, LSE=-inf.
    """
    B, Hh, Npad, D = q.shape
    Nqb = Npad // block
    O = np.full((B, Hh, Npad, D), np.nan)
    LSE = np.full((B, Hh, Npad), np.nan)
    qbs = range(Nqb) if q_blocks is None else q_blocks
    pairs = [(b, h) for b in range(B) for h in range(Hh)] if heads is None else heads
    for b, h in pairs:
        lst = b * Hh + h if per_head else 0
        qh = np.asarray(q[b, h], dtype=np.float64)
        kh = np.asarray(k[b, h], dtype=np.float64)
        vh = np.asarray(v[b, h], dtype=np.float64)
        for qb in qbs:
            r = lst * Nqb + qb
            blocks = np.asarray(col_idx[int(row_ptr[r]):int(row_ptr[r + 1])], dtype=np.int64)
            keys = (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)
            keys = keys[valid[keys]]
            rows = np.arange(qb * block, (qb + 1) * block)
            O[b, h, rows] = 0.0
            LSE[b, h, rows] = -np.inf
            rows = rows[valid[rows]]
            if rows.size == 0 or keys.size == 0:
                continue
            S = (qh[rows] @ kh[keys].T) * scale
            m = S.max(axis=1, keepdims=True)
            p = np.exp(S - m)
            l = p.sum(axis=1, keepdims=True)
            O[b, h, rows] = (p @ vh[keys]) / l
            LSE[b, h, rows] = (m + np.log(l))[:, 0]
    return O, LSE


def attended_pairs(valid: np.ndarray, block: int, row_ptr, col_idx, nlists: int = 1) -> int:
    """Number of (valid query, valid key) pairs a block list admits."""
    nb = valid.size // block
    vcount = valid.reshape(nb, block).sum(axis=1).astype(np.int64)
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    total = 0
    for r in range(nlists * nb):
        qb = r % nb
        total += int(vcount[qb]) * int(vcount[ci[rp[r]:rp[r + 1]]].sum())
    return total


# ---------------------------------------------------------------------------
# FP8 (Draft Attention article, closing paragraph: the authors' next step is
# to bring quantization into Draft Attention).  The article fixes no format;
# the reading taken: Q, K, V in e4m3 (1 sign, 4 exponent bits with bias 7, 3
# mantissa bits, no infinities, largest finite 448), one scale per
# (batch, head) and tensor, scale = fp32(amax) / 448 in fp32 (1 when amax is
# 0), values divided by the scale in fp32 and rounded to the nearest e4m3
# value, ties to even, saturating at +-448.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest e4m3 value (ties to even), saturating at +-448, as fp64.

    Normal e4m3 values in [2^e, 2^(e+1)) (e >= -6) are spaced 2^(e-3);
    below 2^-6 the subnormals are spaced 2^-9.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))       # a = m * 2^ex, m in [0.5, 1)
    quantum = np.where(a >= 2.0 ** -6, np.ldexp(1.0, ex - 1 - 3), 2.0 ** -9)
    r = np.round(a / quantum) * quantum              # np.round: ties to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def fp8_scales(x_nat: np.ndarray) -> np.ndarray:
    """fp32 [B, Hh]: fp32(max |x| over tokens and channels) / 448 (fp32 division)."""
    amax = np.abs(np.asarray(x_nat, dtype=np.float64)).max(axis=(1, 3)).astype(np.float32)
    s = amax / np.float32(E4M3_MAX)
    return np.where(amax == 0, np.float32(1.0), s).astype(np.float32)


def fp8_quantize(x_nat: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """e4m3 codes' values (fp64) of x / scale, the division in fp32: [B, N, Hh, D]."""
    y = np.asarray(x_nat, dtype=np.float32) / scales[:, None, :, None]
    return e4m3_round(y.astype(np.float64))


def fp8_dequantize(q_vals: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The values the fp8 attention computes with: q * scale, fp64 [B, N, Hh, D]."""
    return q_vals * scales.astype(np.float64)[:, None, :, None]
