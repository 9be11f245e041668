"""Pins of the fp64 oracle against what the pages and mathematics fix.

Nothing here retypes an oracle formula: every check is an invariant the pages
state, a closed form derived independently (brute force over candidates, hand
tables, constructed inputs with known answers) or a library routine
(torch scaled_dot_product_attention in float64, math.fsum).
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, make_qkv, small_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# ---------------------------------------------------------------------------
# LVSA ("LVSA: Training-Free Sparse Attention for Long Video Diffusion",
# section 2 "Core mechanism")
# ---------------------------------------------------------------------------

LVSA_CFGS = [(w.T, w.lvsa_C, w.lvsa_T_per) for w in CONFIGS.values() if w.lvsa_C]


def test_anchor_sets_tiny_case_literal():
    # the tiny workload defines G_s = {f : (f - s) mod 4 = 0} on 8 frames
    assert [oracle.lvsa_anchors(8, 4, s) for s in range(4)] == [[0, 4], [1, 5], [2, 6], [3, 7]]
    # Wan-like 6x length: 126 frames, period 12 -> 11 anchors for s < 6, else 10
    assert [len(oracle.lvsa_anchors(126, 12, s)) for s in range(12)] == [11] * 6 + [10] * 6
    assert [len(oracle.lvsa_anchors(65, 16, s)) for s in range(16)] == [5] + [4] * 15


@pytest.mark.parametrize("T,C,T_per", LVSA_CFGS)
def test_every_frame_is_anchor_once_per_period(T, C, T_per):
    # section 2: over T_per consecutive steps every frame is an anchor exactly once
    for s0 in (0, 1, 5, 37):
        hits = np.zeros(T, dtype=int)
        for s in range(s0, s0 + T_per):
            for f in oracle.lvsa_anchors(T, T_per, s):
                hits[f] += 1
        assert (hits == 1).all()


@pytest.mark.parametrize("T,C,T_per", LVSA_CFGS)
def test_frame_set_invariants(T, C, T_per):
    for s in range(T_per):
        G = set(oracle.lvsa_anchors(T, T_per, s))
        A = oracle.lvsa_frame_sets(T, C, T_per, s)
        assert A.shape == (T, C)
        for t in range(T):
            row = list(A[t])
            assert row == sorted(set(row))           # ascending, no repeats
            assert len(row) == C                      # |A(t)| = C (budget)
            assert G <= set(row)                      # anchors always attended
            assert t in row                           # the window is centred on t
            assert all(0 <= f < T for f in row)


def _closed_form(t, T, C, T_per, s):
    """The C - |G U {t}| nearest non-anchor frames, ties to the right."""
    base = {f for f in range(T) if (f - s) % T_per == 0} | {t}
    rest = sorted((f for f in range(T) if f not in base), key=lambda f: (abs(f - t), f < t))
    return sorted(base | set(rest[:C - len(base)]))


def test_window_rule_equals_nearest_non_anchor_closed_form():
    n = 0
    for T in range(1, 13):
        for T_per in range(1, T + 1):
            for s in range(T_per):
                nanch = len([f for f in range(T) if (f - s) % T_per == 0])
                for C in range(1, T + 1):
                    for t in range(T):
                        need = nanch + (0 if (t - s) % T_per == 0 else 1)
                        if need > C:
                            with pytest.raises(ValueError):
                                oracle.lvsa_frame_set(t, T, C, T_per, s, order="distance")
                            continue
                        assert oracle.lvsa_frame_set(t, T, C, T_per, s, order="distance") == \
                            _closed_form(t, T, C, T_per, s), (T, C, T_per, s, t)
                        n += 1
    assert n > 10000


# Hand-derived from the two growth rules for the tiny workload (T=8, C=4,
# T_per=4).  Reading B, the default, follows the workload's own wording: the
# window is extended alternately right then left, skipping anchors, clamped
# at the edges.  E.g. s=0, t=3: G={0,4}, one frame to add; the right pointer
# skips anchor 4 and takes 5 (reading B), while the nearest frame not yet
# present is 2 (reading A, distance order).
HAND_C1_ALTERNATE = {
    0: ["0124", "0124", "0234", "0345", "0345", "0456", "0467", "0467"],
    1: ["0125", "0125", "1235", "1345", "1456", "1456", "1567", "1567"],
    2: ["0126", "1236", "1236", "2346", "2456", "2567", "2567", "2567"],
    3: ["0137", "1237", "2347", "2347", "3457", "3567", "3567", "3567"],
}
HAND_C1_DISTANCE = {
    0: ["0124", "0124", "0234", "0234", "0345", "0456", "0467", "0467"],
    1: ["0125", "0125", "1235", "1345", "1345", "1456", "1567", "1567"],
    2: ["0126", "0126", "1236", "2346", "2456", "2456", "2567", "2567"],
    3: ["0137", "1237", "1237", "2347", "3457", "3567", "3567", "3567"],
}


def _read_golden(name):
    gold = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            s, t, *fr = map(int, line.split())
            gold[(s, t)] = fr
    return gold


@pytest.mark.parametrize("order,hand,golden", [
    ("alternate", HAND_C1_ALTERNATE, "lvsa_tiny_T8_C4_Tper4.txt"),
    ("distance", HAND_C1_DISTANCE, "lvsa_tiny_T8_C4_Tper4_distance.txt")])
def test_tiny_case_hand_table_and_golden(order, hand, golden):
    gold = _read_golden(golden)
    for s, rows in hand.items():
        A = oracle.lvsa_frame_sets(8, 4, 4, s, order=order)
        for t, r in enumerate(rows):
            assert list(A[t]) == [int(c) for c in r], (s, t)
            assert gold[(s, t)] == [int(c) for c in r]
    if order == "alternate":                     # the default
        for s in hand:
            assert (oracle.lvsa_frame_sets(8, 4, 4, s) ==
                    oracle.lvsa_frame_sets(8, 4, 4, s, order=order)).all()


@pytest.mark.parametrize("cid", [1, 3, 4])
def test_lvsa_attended_pairs_is_T_C_P2(cid):
    # section 2 "Complexity": total work T*C*P^2*d, i.e. T*C*P^2 (q, k) pairs
    w = CONFIGS[cid]
    perm, Npad = oracle.frame_layout_perm(w.T, w.H, w.W, w.lvsa_block)
    valid = oracle.slot_valid(perm, Npad)
    nbf = -(-w.P // w.lvsa_block)
    for s in (0, w.lvsa_T_per - 1):
        rp, ci = oracle.lvsa_block_csr(oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s), nbf)
        assert rp[-1] == w.T * nbf * w.lvsa_C * nbf
        assert oracle.attended_pairs(valid, w.lvsa_block, rp, ci) == w.T * w.lvsa_C * w.P ** 2


# ---------------------------------------------------------------------------
# Reorder (Draft Attention article: reorder so that selected blocks are
# contiguous; tiles of pool_h x pool_w = block_size tokens)
# ---------------------------------------------------------------------------


def test_padded_sizes():
    assert oracle.tile_layout_perm(8, 8, 8, 2, 2)[1] == 512
    assert oracle.frame_layout_perm(8, 8, 8, 64)[1] == 512
    assert oracle.tile_layout_perm(21, 30, 52, 8, 16)[1] == 21 * 16 * 128 == 43008
    assert oracle.frame_layout_perm(21, 30, 52, 128)[1] == 21 * 13 * 128
    assert oracle.frame_layout_perm(126, 30, 52, 128)[1] == 209664
    assert oracle.frame_layout_perm(65, 45, 80, 128)[1] == 241280


def test_hand_computed_slots():
    perm, _ = oracle.tile_layout_perm(21, 30, 52, 8, 16)
    n = lambda t, y, x: (t * 30 + y) * 52 + x
    assert perm[n(0, 0, 0)] == 0
    assert perm[n(0, 0, 1)] == 1
    assert perm[n(0, 1, 0)] == 16            # next row of the same 8x16 tile
    assert perm[n(0, 0, 16)] == 128          # next tile to the right
    assert perm[n(0, 29, 51)] == 2003        # tile (3,3), offset (5,3)
    assert perm[n(1, 0, 0)] == 2048          # first tile of frame 1
    perm, _ = oracle.frame_layout_perm(126, 30, 52, 128)
    assert perm[n(0, 29, 51)] == 1559
    assert perm[n(1, 0, 0)] == 1664


@pytest.mark.parametrize("layout", ["tile", "frame"])
def test_reorder_is_bijection_with_zero_pads(layout):
    T, H, W = 3, 10, 13
    if layout == "tile":
        perm, Npad = oracle.tile_layout_perm(T, H, W, 4, 8)
        blk = 32
    else:
        perm, Npad = oracle.frame_layout_perm(T, H, W, 32)
        blk = 32
    assert len(set(perm.tolist())) == T * H * W and perm.min() >= 0 and perm.max() < Npad
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, T * H * W, 3, 8))
    s = oracle.reorder_fwd(x, perm, Npad)
    valid = oracle.slot_valid(perm, Npad)
    assert (s[:, :, ~valid] == 0).all()
    np.testing.assert_array_equal(oracle.reorder_inv(s, perm), x)
    # every block holds tokens of one frame (and one spatial tile)
    for n in range(T * H * W):
        t, y, x_ = n // (H * W), (n // W) % H, n % W
        b = perm[n] // blk
        if layout == "tile":
            TH, TW = -(-H // 4), -(-W // 8)
            assert b == (t * TH + y // 4) * TW + x_ // 8
        else:
            assert b // (-(-H * W // blk)) == t


# ---------------------------------------------------------------------------
# Draft mask (Draft Attention article: average pooling over pool_h x pool_w,
# low-resolution map, top-k blocks at the stated sparsity)
# ---------------------------------------------------------------------------


def test_keep_count():
    assert oracle.draft_keep_count(336, 90) == 34      # 89.88 % actual sparsity
    assert oracle.draft_keep_count(128, 50) == 64
    assert oracle.draft_keep_count(336, 0) == 336
    assert oracle.draft_keep_count(1, 99) == 1
    for nb in range(1, 300):
        for p in (10, 50, 90, 95):
            k = oracle.draft_keep_count(nb, p)
            assert 100 * (nb - k) <= p * nb < 100 * (nb - k + 1)   # never sparser than p


def test_pool_of_constant_ignores_grid_padding():
    # edge tiles hang over the grid (30 % 8 = 6 rows, 52 % 16 = 4 columns);
    # averaging only the tokens inside the grid keeps a constant constant
    T, H, W = 2, 30, 52
    x = np.full((1, T * H * W, 2, 4), 1.5)
    p = oracle.draft_pool(x, T, H, W, 8, 16)
    assert p.shape == (1, 2, 2 * 16, 4)
    assert (p == 1.5).all()


def test_pool_of_ramp_closed_form():
    T, H, W, ph, pw = 1, 30, 52, 8, 16
    yy, xx = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    x = np.stack([yy, xx], -1).reshape(1, H * W, 1, 2).astype(np.float64)
    p = oracle.draft_pool(x, T, H, W, ph, pw)[0, 0]
    for i in range(4):
        for j in range(4):
            ys = [y for y in range(i * ph, min(H, (i + 1) * ph))]
            xs = [v for v in range(j * pw, min(W, (j + 1) * pw))]
            assert p[i * 4 + j, 0] == sum(ys) / len(ys)
            assert p[i * 4 + j, 1] == sum(xs) / len(xs)


def test_pool_matches_exact_mean_within_bound():
    w = small_workload(CONFIGS[2], T=2, Hh=2, D=16, field_grid=(2, 4, 7))
    q, _, _ = make_qkv(w)
    x = q.float().numpy().astype(np.float64)
    p = oracle.draft_pool(x, w.T, w.H, w.W, 8, 16)
    xr = x.reshape(1, w.T, w.H, w.W, w.Hh, w.D)
    eps = 2.0 ** -53
    for t in range(w.T):
        for i in range(4):
            for j in range(4):
                tile = xr[0, t, i * 8:(i + 1) * 8, j * 16:(j + 1) * 16]
                n = tile.shape[0] * tile.shape[1]
                for h in range(w.Hh):
                    for c in range(w.D):
                        vals = tile[:, :, h, c].reshape(-1)
                        exact = math.fsum(vals) / n
                        bound = (n + 1) * eps * np.abs(vals).sum() / n
                        assert abs(p[0, h, (t * 4 + i) * 4 + j, c] - exact) <= bound


def test_one_block_covers_the_frame():
    # pool over the whole frame: a single block, which top-k must keep
    T, H, W = 1, 4, 6
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, T * H * W, 1, 8))
    k = rng.standard_normal((1, T * H * W, 1, 8))
    blocks = oracle.draft_blocks(q, k, T, H, W, H, W, 90)
    assert blocks.shape == (1, 1, 1, 1) and blocks[0, 0, 0, 0] == 0
    np.testing.assert_allclose(oracle.draft_pool(q, T, H, W, H, W)[0, 0, 0], q[0, :, 0].mean(0),
                               rtol=1e-14, atol=1e-15)


def _constructed_qk():
    """Tokens of block i carry query w_i, of block j key u_j (small integers)."""
    T, H, W, ph, pw = 1, 4, 4, 2, 2          # 4 blocks of 4 tokens
    Wq = np.array([[1, 0, 2], [0, 3, 0], [2, 1, 0], [0, 0, 1]], dtype=np.float64)
    Uk = np.array([[0, 1, 0], [4, 0, 0], [0, 0, 3], [1, 2, 1]], dtype=np.float64)
    q = np.zeros((1, 16, 1, 3))
    k = np.zeros((1, 16, 1, 3))
    for y in range(H):
        for x in range(W):
            b = (y // 2) * 2 + x // 2
            q[0, y * W + x, 0] = Wq[b]
            k[0, y * W + x, 0] = Uk[b]
    return q, k, T, H, W, ph, pw


def test_logits_and_topk_on_constructed_input():
    q, k, T, H, W, ph, pw = _constructed_qk()
    L = oracle.draft_logits(oracle.draft_pool(q, T, H, W, ph, pw),
                            oracle.draft_pool(k, T, H, W, ph, pw))[0, 0]
    # L[i][j] = <w_i, u_j>, by hand
    expect = np.array([[0, 4, 6, 3],
                       [3, 0, 0, 6],
                       [1, 8, 0, 4],
                       [0, 0, 3, 1]], dtype=np.float64)
    np.testing.assert_array_equal(L, expect)
    top1 = oracle.draft_blocks(q, k, T, H, W, ph, pw, 75)[0, 0, :, 0]
    assert list(top1) == [2, 3, 1, 2]          # row-wise argmax (not column-wise)
    top2 = oracle.draft_blocks(q, k, T, H, W, ph, pw, 50)[0, 0]
    assert [list(r) for r in top2] == [[1, 2], [0, 3], [1, 3], [2, 3]]


def test_topk_ties_go_to_lower_index_and_bruteforce():
    rng = np.random.default_rng(5)
    L = rng.integers(-3, 4, size=(2, 3, 7, 9)).astype(np.float64)   # many ties
    for k in (1, 3, 9):
        got = oracle.draft_topk(L, k)
        for idx in itertools.product(range(2), range(3), range(7)):
            row = L[idx]
            best = sorted(range(9), key=lambda j: (-row[j], j))[:k]
            assert list(got[idx]) == sorted(best)
    assert (oracle.draft_topk(L, 9) == np.arange(9)).all()


def test_logits_match_library_dot():
    rng = np.random.default_rng(7)
    a = rng.standard_normal((1, 2, 11, 32))
    b = rng.standard_normal((1, 2, 13, 32))
    np.testing.assert_allclose(oracle.draft_logits(a, b), np.einsum("bhic,bhjc->bhij", a, b),
                               rtol=1e-13, atol=1e-13)


def test_logits_match_library_dot_within_the_fp32_bound():
    # Recursive summation of D rounded products: |fl(L) - L| <= gamma_D *
    # sum_c |q_c k_c| with gamma_D = D u / (1 - D u), u = 2^-24 (Higham,
    # "Accuracy and Stability of Numerical Algorithms", section 3.1), L the
    # exact dot product of the fp32-rounded pooled values.
    rng = np.random.default_rng(7)
    a = rng.standard_normal((1, 2, 11, 32))
    b = rng.standard_normal((1, 2, 13, 32))
    got = oracle.draft_logits(a, b, "fp32")
    assert got.dtype == np.float32
    a32, b32 = (x.astype(np.float32).astype(np.float64) for x in (a, b))
    exact = np.einsum("bhic,bhjc->bhij", a32, b32)
    u = 2.0 ** -24
    gamma = 32 * u / (1 - 32 * u)
    bound = gamma * np.einsum("bhic,bhjc->bhij", np.abs(a32), np.abs(b32))
    assert (np.abs(got.astype(np.float64) - exact) <= bound).all()
    # and it is not the fp64 chain: some logit differs from it
    assert (got.astype(np.float64) != oracle.draft_logits(a, b)).any()


# ---------------------------------------------------------------------------
# Block-sparse attention (the sparse mask guides full-resolution softmax
# attention; a full mask is dense attention)
# ---------------------------------------------------------------------------


def _sdpa64(q, k, v, mask, scale):
    """torch SDPA in float64 on CPU: [Hh, L, D] with bool mask [L, S]."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask), scale=scale).numpy()


def test_full_mask_is_dense_attention_tiny_workload():
    w = CONFIGS[1]
    q, k, v = (t.float().numpy().astype(np.float64) for t in make_qkv(w))
    perm, Npad = oracle.frame_layout_perm(w.T, w.H, w.W, 64)
    valid = oracle.slot_valid(perm, Npad)
    rp, ci = oracle.dense_block_csr(Npad // 64)
    qs, ks, vs = (oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v))
    O, LSE = oracle.masked_attention(qs, ks, vs, valid, 64, rp, ci, False, 1 / 8.0)
    On = oracle.reorder_inv(O, perm)
    ref = _sdpa64(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2), v[0].transpose(1, 0, 2),
                  np.ones((w.N, w.N), bool), 1 / 8.0)
    np.testing.assert_allclose(On[0].transpose(1, 0, 2), ref, rtol=1e-12, atol=1e-12)
    # LSE by its definition, with an exactly rounded sum
    for h, n in ((0, 0), (1, 77), (0, 511)):
        sc = [float(q[0, n, h] @ k[0, m, h]) / 8.0 for m in range(w.N)]
        mx = max(sc)
        ref_lse = mx + math.log(math.fsum(math.exp(s - mx) for s in sc))
        assert abs(LSE[0, h, perm[n]] - ref_lse) < 1e-11


def test_padded_tile_layout_dense_matches_sdpa():
    # grid edges leave empty slots: they must never be attended or reported
    T, H, W, ph, pw, D = 2, 5, 7, 4, 4, 16
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, D)) for _ in range(3))
    perm, Npad = oracle.tile_layout_perm(T, H, W, ph, pw)
    valid = oracle.slot_valid(perm, Npad)
    rp, ci = oracle.dense_block_csr(Npad // 16)
    O, LSE = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v)),
                                     valid, 16, rp, ci, False, 0.25)
    assert (O[:, :, ~valid] == 0).all() and np.isneginf(LSE[:, :, ~valid]).all()
    ref = _sdpa64(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2), v[0].transpose(1, 0, 2),
                  np.ones((T * H * W,) * 2, bool), 0.25)
    np.testing.assert_allclose(oracle.reorder_inv(O, perm)[0].transpose(1, 0, 2), ref,
                               rtol=1e-12, atol=1e-12)


def test_lvsa_mask_attention_matches_sdpa_with_frame_mask():
    # the frame mask built straight from A(t): query frame t sees frames A(t)
    w = CONFIGS[1]
    q, k, v = (t.float().numpy().astype(np.float64) for t in make_qkv(w))
    perm, Npad = oracle.frame_layout_perm(w.T, w.H, w.W, 64)
    valid = oracle.slot_valid(perm, Npad)
    for s in range(4):
        A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s)
        rp, ci = oracle.lvsa_block_csr(A, 1)
        O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v)),
                                       valid, 64, rp, ci, False, 1 / 8.0)
        frame = np.arange(w.N) // w.P
        allowed = np.zeros((w.T, w.T), bool)
        for t in range(w.T):
            allowed[t, HAND_C1_SETS[s][t]] = True         # reading B, the default
        mask = allowed[frame[:, None], frame[None, :]]
        ref = _sdpa64(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                      v[0].transpose(1, 0, 2), mask, 1 / 8.0)
        np.testing.assert_allclose(oracle.reorder_inv(O, perm)[0].transpose(1, 0, 2), ref,
                                   rtol=1e-12, atol=1e-12)


HAND_C1_SETS = {s: [[int(c) for c in r] for r in rows] for s, rows in HAND_C1_ALTERNATE.items()}


def test_draft_mask_attention_matches_sdpa_with_block_mask():
    T, H, W, ph, pw, D = 2, 6, 8, 2, 4, 8
    rng = np.random.default_rng(13)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, D)) for _ in range(3))
    kv = oracle.draft_blocks(q, k, T, H, W, ph, pw, 60)
    rp, ci = oracle.fixed_k_csr(kv)
    perm, Npad = oracle.tile_layout_perm(T, H, W, ph, pw)
    valid = oracle.slot_valid(perm, Npad)
    O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v)),
                                   valid, ph * pw, rp, ci, True, 0.3)
    On = oracle.reorder_inv(O, perm)
    blk_of = perm // (ph * pw)
    for h in range(2):
        allowed = np.zeros((Npad // 8,) * 2, bool)
        for i in range(kv.shape[2]):
            allowed[i, kv[0, h, i]] = True
        mask = allowed[blk_of[:, None], blk_of[None, :]]
        ref = _sdpa64(q[0, :, h][None], k[0, :, h][None], v[0, :, h][None], mask, 0.3)[0]
        np.testing.assert_allclose(On[0, :, h], ref, rtol=1e-12, atol=1e-12)


def test_constant_values_and_single_key_and_empty_row():
    rng = np.random.default_rng(17)
    B, Hh, Npad, D, blk = 1, 1, 8, 4, 2
    q = rng.standard_normal((B, Hh, Npad, D))
    k = rng.standard_normal((B, Hh, Npad, D))
    v = np.tile(np.array([0.5, -2.0, 3.0, 7.0]), (B, Hh, Npad, 1))
    valid = np.ones(Npad, bool)
    valid[7] = False                            # one empty slot in the last block
    rp = np.array([0, 2, 3, 3, 4], np.int32)    # rows: {0,1}, {3}, {}, {3}
    ci = np.array([0, 1, 3, 3], np.int32)
    O, LSE = oracle.masked_attention(q, k, v, valid, blk, rp, ci, False, 0.5)
    np.testing.assert_allclose(O[0, 0, :4], v[0, 0, :4], rtol=0, atol=1e-15)   # constant V
    # block 1 sees only block 3, whose single valid key is slot 6
    v2 = rng.standard_normal((B, Hh, Npad, D))
    O2, LSE2 = oracle.masked_attention(q, k, v2, valid, blk, rp, ci, False, 0.5)
    for r in (2, 3):
        np.testing.assert_allclose(O2[0, 0, r], v2[0, 0, 6], rtol=1e-15, atol=1e-15)
        assert abs(LSE2[0, 0, r] - 0.5 * float(q[0, 0, r] @ k[0, 0, 6])) < 1e-14
    # block 2 has an empty row; slot 7 is padding
    assert (O2[0, 0, 4:6] == 0).all() and np.isneginf(LSE2[0, 0, 4:6]).all()
    assert (O2[0, 0, 7] == 0).all() and np.isneginf(LSE2[0, 0, 7])
    np.testing.assert_allclose(O2[0, 0, 6], v2[0, 0, 6], rtol=1e-15, atol=1e-15)


def test_output_does_not_depend_on_layout():
    # same tokens, same dense mask, two layouts -> the same natural-order output
    T, H, W, D = 2, 6, 10, 8
    rng = np.random.default_rng(19)
    q, k, v = (rng.standard_normal((1, T * H * W, 1, D)) for _ in range(3))
    outs = []
    for perm, Npad, blk in ((*oracle.tile_layout_perm(T, H, W, 4, 4), 16),
                            (*oracle.frame_layout_perm(T, H, W, 16), 16)):
        valid = oracle.slot_valid(perm, Npad)
        rp, ci = oracle.dense_block_csr(Npad // blk)
        O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v)),
                                       valid, blk, rp, ci, False, 0.35)
        outs.append(oracle.reorder_inv(O, perm))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------------
# Mask variants: fixed-grid anchors and the sliding window (LVSA, section 2:
# the fixed grid that rotating anchors replace; the introduction's sliding
# window), window growth reading B, max pooling (Draft Attention article: the
# max pooling tried before average pooling)
# ---------------------------------------------------------------------------


def test_fixed_grid_anchors_do_not_move_with_the_step():
    for T, C, T_per in LVSA_CFGS:
        G = [f for f in range(0, T, T_per)]          # every T_per-th frame from 0
        for s in range(T_per):
            assert oracle.lvsa_anchors(T, T_per, s, "fixed") == G
        A0 = oracle.lvsa_frame_sets(T, C, T_per, 0, anchors="fixed")
        for s in (1, T_per - 1):
            assert (oracle.lvsa_frame_sets(T, C, T_per, s, anchors="fixed") == A0).all()


@pytest.mark.parametrize("order", ["distance", "alternate"])
def test_window_only_is_a_clamped_interval(order):
    # with no anchors the C frames nearest t (ties to the right) are the
    # interval [lo, lo + C - 1], lo = t - floor((C - 1) / 2) clamped into
    # [0, T - C]; both growth orders give it (the sides alternate either way)
    for T in range(1, 14):
        for C in range(1, T + 1):
            for t in range(T):
                lo = min(max(t - (C - 1) // 2, 0), T - C)
                got = oracle.lvsa_frame_set(t, T, C, 1, 0, anchors="none", order=order)
                assert got == list(range(lo, lo + C)), (T, C, t)


def test_alternate_order_hand_case():
    # T = 8, C = 4, T_per = 4, s = 0, t = 3: G = {0, 4}, one frame to add.
    # distance order tries +1 = 4 (already there), then -1 = 2;
    # alternate order moves the right pointer past 4 and takes 5.
    assert oracle.lvsa_frame_set(3, 8, 4, 4, 0, order="distance") == [0, 2, 3, 4]
    assert oracle.lvsa_frame_set(3, 8, 4, 4, 0, order="alternate") == [0, 3, 4, 5]
    assert oracle.lvsa_frame_set(3, 8, 4, 4, 0) == [0, 3, 4, 5]          # the default


def test_alternate_order_closed_form():
    # reading B as a count: with need = C - |G U {t}| frames to add and nR / nL
    # frames outside G U {t} right / left of t, the right side takes
    # kR = min(nR, max(ceil(need/2), need - nL)) of its nearest frames and the
    # left side the remaining need - kR of its own
    for T in range(1, 13):
        for T_per in range(1, T + 2):
            for s in range(T_per):
                for anchors in ("rotating", "none"):
                    G = set(oracle.lvsa_anchors(T, T_per, s, anchors))
                    for t in range(T):
                        base = G | {t}
                        right = [f for f in range(t + 1, T) if f not in base]
                        left = [f for f in range(t - 1, -1, -1) if f not in base]
                        for C in range(len(base), T + 1):
                            need = C - len(base)
                            kR = min(len(right), max((need + 1) // 2, need - len(left)))
                            want = sorted(base | set(right[:kR]) | set(left[:need - kR]))
                            got = oracle.lvsa_frame_set(t, T, C, T_per, s, anchors, "alternate")
                            assert got == want, (T, T_per, s, t, C, anchors)


@pytest.mark.parametrize("anchors", ["fixed", "none"])
def test_variant_invariants(anchors):
    for T, C, T_per in LVSA_CFGS:
        for s in (0, 1):
            G = set(oracle.lvsa_anchors(T, T_per, s, anchors))
            for order in ("distance", "alternate"):
                A = oracle.lvsa_frame_sets(T, C, T_per, s, anchors, order)
                for t in range(T):
                    row = list(A[t])
                    assert row == sorted(set(row)) and len(row) == C
                    assert G <= set(row) and t in row


def test_max_pool_closed_forms():
    T, H, W, ph, pw = 1, 30, 52, 8, 16
    # constant: the constant; ramp: the largest coordinate inside the grid
    x = np.full((1, T * H * W, 1, 3), -2.25)
    assert (oracle.draft_pool(x, T, H, W, ph, pw, "max") == -2.25).all()
    yy, xx = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    r = np.stack([yy, xx], -1).reshape(1, H * W, 1, 2).astype(np.float64)
    p = oracle.draft_pool(r, T, H, W, ph, pw, "max")[0, 0]
    for i in range(4):
        for j in range(4):
            assert p[i * 4 + j, 0] == min(H, (i + 1) * ph) - 1
            assert p[i * 4 + j, 1] == min(W, (j + 1) * pw) - 1


def test_max_pool_brute_force_and_bounds_mean():
    w = small_workload(CONFIGS[2], T=2, Hh=2, D=8, field_grid=(2, 4, 7))
    q, _, _ = make_qkv(w)
    x = q.float().numpy().astype(np.float64)
    mx = oracle.draft_pool(x, w.T, w.H, w.W, 8, 16, "max")
    mean = oracle.draft_pool(x, w.T, w.H, w.W, 8, 16, "mean")
    assert (mx >= mean).all()
    xr = x.reshape(1, w.T, w.H, w.W, w.Hh, w.D)
    for t in range(w.T):
        for i in range(4):
            for j in range(4):
                tile = xr[0, t, i * 8:(i + 1) * 8, j * 16:(j + 1) * 16]
                for h in range(w.Hh):
                    for c in range(w.D):
                        vals = sorted(tile[:, :, h, c].reshape(-1).tolist())
                        assert mx[0, h, (t * 4 + i) * 4 + j, c] == vals[-1]


# ---------------------------------------------------------------------------
# FP8 e4m3 (Draft Attention article: quantization as the next step)
# ---------------------------------------------------------------------------


def test_e4m3_grid_is_every_finite_bit_pattern():
    # torch's float8_e4m3fn decoding of all 256 codes is the library reference
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    vals = codes.to(torch.float64).numpy()
    fin = np.isfinite(vals)
    assert fin.sum() == 254                      # 0x7f and 0xff are NaN
    assert np.array_equal(oracle.e4m3_round(vals[fin]), vals[fin])   # the grid maps to itself
    assert vals[fin].max() == 448.0 and sorted(set(np.abs(vals[fin])))[1] == 2.0 ** -9


def test_e4m3_round_matches_library_cast():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 60, 20000),
                        rng.uniform(-464, 464, 20000), rng.normal(0, 2.0 ** -8, 20000),
                        np.ldexp(rng.integers(-64, 64, 4000) + 0.5, -10)])   # exact ties
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(x), ref)
    # beyond the largest finite value the rounding saturates
    assert (oracle.e4m3_round(np.array([480.0, 1e6, -1e9])) == [448.0, 448.0, -448.0]).all()


def test_fp8_scales_and_quantize():
    rng = np.random.default_rng(6)
    x = rng.normal(0, 1, (2, 40, 3, 16)).astype(np.float32).astype(np.float64)
    x[1, :, 2] = 0.0                                    # an all-zero head: scale 1
    s = oracle.fp8_scales(x)
    assert s.dtype == np.float32 and s[1, 2] == 1.0
    amax = np.abs(x).max(axis=(1, 3)).astype(np.float32)
    assert s[0, 0] == np.float32(amax[0, 0]) / np.float32(448.0)
    q = oracle.fp8_quantize(x, s)
    # the largest |x| of a head lands on +-448 (within the fp32 division's rounding)
    qmax = np.abs(q).max(axis=(1, 3))
    assert (qmax[s != 1.0] >= 416.0).all() and (qmax <= 448.0).all()
    # values are on the e4m3 grid, and dequantized values are within half a step
    assert np.array_equal(oracle.e4m3_round(q), q)
    deq = oracle.fp8_dequantize(q, s)
    step = np.maximum(np.ldexp(1.0, np.frexp(np.abs(q) + 1e-300)[1] - 4), 2.0 ** -9)
    assert (np.abs(deq - x) <= 0.5 * step * s.astype(np.float64)[:, None, :, None] * (1 + 1e-6)
            + 1e-12).all()


def test_fp8_quantize_is_exact_for_values_on_the_grid_with_power_of_two_scales():
    # amax 448 * 2^-5 gives scale 2^-5 exactly; e4m3 values times 2^-5 survive
    grid = oracle.e4m3_round(np.linspace(-448, 448, 301))
    x = (grid * 2.0 ** -5).reshape(1, 301, 1, 1)
    s = oracle.fp8_scales(x)
    assert s[0, 0] == np.float32(2.0 ** -5)
    np.testing.assert_array_equal(oracle.fp8_dequantize(oracle.fp8_quantize(x, s), s), x)


# ---------------------------------------------------------------------------
# The draft attention map (Draft Attention article: the low-resolution
# attention map softmax(Qbar Kbar^T / sqrt(D)) of the pooled queries and
# keys), the fp64 evaluation order the selection follows, and the LVSA block
# list at several blocks per frame
# ---------------------------------------------------------------------------


def test_draft_map_matches_library_softmax_over_key_blocks():
    rng = np.random.default_rng(23)
    D = 64
    L = rng.standard_normal((2, 3, 7, 11)) * 9.0
    got = oracle.draft_map(L, D)
    ref = torch.softmax(torch.from_numpy(L) / math.sqrt(D), dim=-1).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-16)
    # a distribution over key blocks for every query block, not over queries
    np.testing.assert_allclose(got.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    assert not np.allclose(got.sum(axis=-2), 1.0)


def test_draft_map_hand_cases():
    D = 128
    # equal logits: uniform over the Nb key blocks
    L = np.full((1, 1, 3, 5), 2.5)
    np.testing.assert_allclose(oracle.draft_map(L, D), 0.2, rtol=0, atol=1e-16)
    # one logit ahead by delta*sqrt(D): weight ratio exp(delta), so with Nb
    # blocks the leader holds e^delta / (e^delta + Nb - 1)
    for delta in (0.5, 1.0, 3.0):
        row = np.zeros((1, 1, 1, 4))
        row[..., 2] = delta * math.sqrt(D)
        m = oracle.draft_map(row, D)[0, 0, 0]
        assert m[2] / m[0] == pytest.approx(math.exp(delta), rel=1e-13)
        assert m[2] == pytest.approx(math.exp(delta) / (math.exp(delta) + 3), rel=1e-13)
    # a shift of a whole row changes nothing; scaling by sqrt(D) is applied once
    L = np.array([[[[0.0, math.sqrt(D) * math.log(3.0)]]]])
    np.testing.assert_allclose(oracle.draft_map(L, D)[0, 0, 0], [0.25, 0.75], rtol=1e-14)
    np.testing.assert_allclose(oracle.draft_map(L + 1e3, D), oracle.draft_map(L, D), rtol=1e-12)


def test_pool_sums_in_row_major_order():
    # one 2 x 2 tile whose sum depends on the order: row-major (a, then b)
    # adds 2^-53 + 2^-53 = 2^-52 before the 1, which then survives; the
    # column-major order adds 2^-53 to 1 first, which rounds away.
    T, H, W, ph, pw = 1, 2, 2, 2, 2
    x = np.zeros((1, 4, 1, 1))
    x[0, 0, 0, 0] = 2.0 ** -53        # (a, b) = (0, 0)
    x[0, 1, 0, 0] = 2.0 ** -53        # (0, 1)
    x[0, 2, 0, 0] = 1.0               # (1, 0)
    x[0, 3, 0, 0] = 0.0               # (1, 1)
    got = oracle.draft_pool(x, T, H, W, ph, pw)[0, 0, 0, 0]
    assert got == (1.0 + 2.0 ** -52) / 4
    assert ((2.0 ** -53 + 1.0) + 2.0 ** -53) / 4 != got     # the other order differs


def test_fp32_and_fp64_logits_within_the_certification_bound():
    # The GPU takes the fp64 draft lists from fp32 logits wherever they are
    # further than twice e = c |q| max|k| + 2^-100 from the k-th logit, with
    # c = 2 (gamma_D(fp32) (1 + u32)^2 + 2 u32 + u32^2 + gamma_D(fp64)),
    # gamma_n = n u / (1 - n u) (Higham, "Accuracy and Stability of Numerical
    # Algorithms", sections 3.1 and 3.5).  The two oracles' logits must be
    # that close on every pair, here on random rows, on rows spread over
    # many binades, and on nearly cancelling rows.
    rng = np.random.default_rng(17)
    D = 128
    u32, u64 = 2.0 ** -24, 2.0 ** -53
    g32, g64 = D * u32 / (1 - D * u32), D * u64 / (1 - D * u64)
    c = 2.0 * (g32 * (1 + u32) ** 2 + 2 * u32 + u32 * u32 + g64)
    cases = [rng.standard_normal((2, 40, D)),
             rng.standard_normal((2, 40, D)) * np.exp2(rng.integers(-30, 30, size=(2, 40, D)))]
    base = rng.standard_normal((1, 40, D))
    cases.append(np.concatenate([base, -base + 1e-7 * rng.standard_normal((1, 40, D))]))
    for x in cases:
        q, k = x[0][None, None], x[1][None, None]
        L64 = oracle.draft_logits(q, k)[0, 0]
        L32 = oracle.draft_logits(q, k, "fp32")[0, 0].astype(np.float64)
        qn = np.sqrt((x[0] ** 2).sum(-1))
        kn = np.sqrt((x[1] ** 2).sum(-1))
        e = c * qn[:, None] * kn.max() + 2.0 ** -100
        assert (np.abs(L32 - L64) <= e).all()
        assert (np.abs(L32 - L64) <= c * qn[:, None] * kn[None, :] + 2.0 ** -100).all()
        assert (L32 != L64).any()      # the precisions do differ


def test_logits_are_sequential_and_unfused():
    # channel 0 first: acc = -(1 + 2^-29); channel 1 adds the rounded product
    # x*x with x = 1 + 2^-30, i.e. 1 + 2^-29 (the exact square carries an
    # extra 2^-60), so the sum is exactly 0.  A fused multiply-add would keep
    # 2^-60; the reversed order would give the same 0 here, so a second
    # case pins the order: 1, then 2^-53 twice, rounds back to 1 each time.
    x = 1.0 + 2.0 ** -30
    q = np.array([1.0, x]).reshape(1, 1, 1, 2)
    k = np.array([-(1.0 + 2.0 ** -29), x]).reshape(1, 1, 1, 2)
    assert oracle.draft_logits(q, k)[0, 0, 0, 0] == 0.0
    # the exact value a fused multiply-add would round: 2^-60, not 0
    assert Fraction(x) * Fraction(x) - Fraction(1.0 + 2.0 ** -29) == Fraction(1, 2 ** 60)
    q = np.ones((1, 1, 1, 3))
    k = np.array([1.0, 2.0 ** -53, 2.0 ** -53]).reshape(1, 1, 1, 3)
    assert oracle.draft_logits(q, k)[0, 0, 0, 0] == 1.0                 # c = 0, 1, 2
    assert (2.0 ** -53 + 2.0 ** -53) + 1.0 == 1.0 + 2.0 ** -52           # reversed differs


def test_logits_are_fp32_sequential_and_unfused():
    # channel 0 first: acc = -(1 + 2^-11); channel 1 adds the rounded product
    # x*x with x = 1 + 2^-12: the exact square 1 + 2^-11 + 2^-24 lies half an
    # fp32 ulp above 1 + 2^-11 and rounds to it (ties to even), so the sum is
    # exactly 0.  A fused multiply-add would keep 2^-24.
    x = 1.0 + 2.0 ** -12
    assert Fraction(x) * Fraction(x) - Fraction(1.0 + 2.0 ** -11) == Fraction(1, 2 ** 24)
    q = np.array([1.0, x]).reshape(1, 1, 1, 2)
    k = np.array([-(1.0 + 2.0 ** -11), x]).reshape(1, 1, 1, 2)
    assert oracle.draft_logits(q, k, "fp32")[0, 0, 0, 0] == 0.0
    # the products are rounded to fp32, not fp64: x*x alone
    one = oracle.draft_logits(np.array([x]).reshape(1, 1, 1, 1), np.array([x]).reshape(1, 1, 1, 1), "fp32")
    assert one[0, 0, 0, 0] == 1.0 + 2.0 ** -11 and x * x != 1.0 + 2.0 ** -11
    # order: 1, then 2^-24 twice, rounds back to 1 each time (half an ulp,
    # ties to even); the reversed order gives 1 + 2^-23
    q = np.ones((1, 1, 1, 3))
    k = np.array([1.0, 2.0 ** -24, 2.0 ** -24]).reshape(1, 1, 1, 3)
    assert oracle.draft_logits(q, k, "fp32")[0, 0, 0, 0] == 1.0
    assert np.float32(np.float32(2.0 ** -24) + np.float32(2.0 ** -24)) + np.float32(1.0) == \
        np.float32(1.0 + 2.0 ** -23)
    # the pooled values are rounded to the nearest fp32 before the products:
    # 1 + 3*2^-25 is 0.75 ulp above 1 and rounds up, 1 + 2^-30 rounds down
    ones = np.ones((1, 1, 1, 1))
    assert oracle.draft_logits(np.full((1, 1, 1, 1), 1.0 + 3 * 2.0 ** -25), ones, "fp32")[0, 0, 0, 0] == \
        1.0 + 2.0 ** -23
    assert oracle.draft_logits(np.full((1, 1, 1, 1), 1.0 + 2.0 ** -30), ones, "fp32")[0, 0, 0, 0] == 1.0


def test_lvsa_block_csr_literal_table_two_blocks_per_frame():
    # T=3, C=2, T_per=3, s=0: G={0}; A(0)={0,1}, A(1)={0,1}, A(2)={0,2}.
    # Two blocks per frame: frame f owns blocks 2f and 2f+1, and both query
    # blocks of a frame carry that frame's list.
    A = oracle.lvsa_frame_sets(3, 2, 3, 0)
    assert A.tolist() == [[0, 1], [0, 1], [0, 2]]
    rp, ci = oracle.lvsa_block_csr(A, 2)
    assert rp.tolist() == [0, 4, 8, 12, 16, 20, 24]
    rows = [ci[rp[r]:rp[r + 1]].tolist() for r in range(6)]
    assert rows == [[0, 1, 2, 3], [0, 1, 2, 3], [0, 1, 2, 3], [0, 1, 2, 3],
                    [0, 1, 4, 5], [0, 1, 4, 5]]
    # three blocks per frame, frame sets of a later step
    A = oracle.lvsa_frame_sets(3, 2, 3, 2)          # G={2}: A = {0,2}, {1,2}, {1,2}
    assert A.tolist() == [[0, 2], [1, 2], [1, 2]]
    rp, ci = oracle.lvsa_block_csr(A, 3)
    assert ci[rp[0]:rp[1]].tolist() == [0, 1, 2, 6, 7, 8]
    assert ci[rp[5]:rp[6]].tolist() == [3, 4, 5, 6, 7, 8]
    assert ci[rp[8]:rp[9]].tolist() == [3, 4, 5, 6, 7, 8]


@pytest.mark.parametrize("order", ["alternate", "distance"])
def test_lvsa_csr_attention_matches_sdpa_with_several_blocks_per_frame(order):
    # frames of 15 tokens on 4-token blocks: 4 blocks per frame, the last one
    # holding 3 tokens and one empty slot; the token mask comes straight from
    # the frame sets, not from the block list
    T, H, W, D, blk, C, T_per = 6, 3, 5, 8, 4, 3, 4
    P = H * W
    rng = np.random.default_rng(29)
    q, k, v = (rng.standard_normal((1, T * P, 2, D)) for _ in range(3))
    perm, Npad = oracle.frame_layout_perm(T, H, W, blk)
    nbf = Npad // (T * blk)
    assert nbf == 4
    valid = oracle.slot_valid(perm, Npad)
    for s in range(T_per):
        A = oracle.lvsa_frame_sets(T, C, T_per, s, order=order)
        rp, ci = oracle.lvsa_block_csr(A, nbf)
        O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Npad) for x in (q, k, v)),
                                       valid, blk, rp, ci, False, 0.35)
        frame = np.arange(T * P) // P
        allowed = np.zeros((T, T), bool)
        for t in range(T):
            allowed[t, A[t]] = True
        mask = allowed[frame[:, None], frame[None, :]]
        ref = _sdpa64(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2),
                      v[0].transpose(1, 0, 2), mask, 0.35)
        np.testing.assert_allclose(oracle.reorder_inv(O, perm)[0].transpose(1, 0, 2), ref,
                                   rtol=1e-12, atol=1e-12)
